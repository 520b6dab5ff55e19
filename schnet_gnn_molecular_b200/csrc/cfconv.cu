// Fused continuous-filter convolution on the sm_100a tensor cores.
//
// One kernel per interaction and direction does, for 128-edge tiles of a CTA's
// contiguous CSR rows:
//   flash radial basis  (FlashSchNet paper-curation summary, How): distance,
//     Gaussian expansion and cosine envelope computed once per edge into
//     shared memory, never to HBM;
//   filter network      (How, quantization item; contraction on tensor cores):
//     W(d) = f_c(d) (ssp(e W1 + b1) W2 + b2) as two chained tcgen05 GEMMs with
//     TMEM accumulators; channel-wise scaled 16-bit operands, hi/lo split of
//     the activations (and of fp32-stored weights) with fp32 accumulation;
//   flash message passing + flash aggregation (How): cutoff masking, gather of
//     h_j, filter product and the CSR segment sum m_i = sum_j h_j (.) W_ij,
//     accumulated in registers, no atomics, no edge tensor in HBM.
// The backward kernel recomputes W and its distance derivative W' by forward-
// mode tangents and produces dE/dh_j (segment sum over the symmetric list) and
// the per-edge scalar s_e = sum_f W'_f u_i,f h_j,f (the edge's share of dE/dd).
//
// Tile orientation: the GEMMs are computed transposed, D[f][e] = W^T[f][k] B[e][k],
// so TMEM lane = output feature and TMEM column = edge.  Each epilogue thread
// then owns one feature of every edge in the tile, the per-row reduction is a
// running sum in one register, and the h_j gathers are 512-byte coalesced rows.
#include "internal.h"

namespace schnet {

struct MPArgs {
    const float4* pos4;
    const int32_t* crow;     // compacted edges (d < r_c) of each CTA's rows: row, column,
    const int32_t* ccol;     //   and index in the full list; CTA c's run starts at
    const int32_t* cidx;     //   row_ptr[part[c]] and holds ccount[c] edges
    const int32_t* ccount;
    const int32_t* row_ptr;
    const int32_t* part;
    DevMeta* meta;
    long long cap;
    Box box;
    float rc, inv_rc;
    float mu0, dmu;       // Gaussian centres mu_k = mu0 + k dmu
    float ngc;            // -log2(e) / (2 sigma^2): e_k = 2^(ngc (d - mu_k)^2)
    const uint8_t* img;   // this layer's packed W1^T / W2^T images
    const float *s1, *s2, *b1;  // this layer's channel scales and first-layer bias [FP]
    const float* b2s;     // second-layer bias folded with the base-2 softplus shift [FP]
    const float* h;       // [N][FP]
    const float* u;       // [N][FP]   (backward)
    float* out;           // m (forward) or dh (backward)   [N][FP]
    float* s_edge;        // [cap]     (backward)
    int accumulate_s;
};

constexpr int NT = 512;   // threads per CTA: 16 warps, four per TMEM lane quadrant

// shared-memory map (bytes)
constexpr uint32_t SM_W1 = 0;                          // W1^T hi, lo   2 x 16 KB
constexpr uint32_t SM_W2 = 32768;                      // W2^T hi, lo   2 x 32 KB
constexpr uint32_t SM_X = 98304;                       // fwd: rbf hi/lo (32 KB) ; bwd: rbf, rbf' then a (64 KB)
constexpr uint32_t SM_FWD_A = 131072;                  // fwd: a hi/lo (64 KB)
constexpr uint32_t SM_BWD_Y = 163840;                  // bwd: ssp'(p) p' hi/lo (64 KB); partial sums after GEMM2
constexpr uint32_t SM_META_FWD = 196608;
constexpr uint32_t SM_META_BWD = 229376;
constexpr uint32_t TILEMETA_BYTES = 2048 + 64;         // per-edge records + per-chunk row summary
constexpr uint32_t PART_BYTES = 2 * 4 * 128 * 4;       // first/last-row partial per chunk and feature
// forward: two metadata buffers (tile t and the next tile are live together)
constexpr uint32_t SMEM_FWD = SM_META_FWD + 2 * TILEMETA_BYTES + PART_BYTES + 16;
constexpr uint32_t SMEM_BWD = SM_META_BWD + TILEMETA_BYTES + 16;
static_assert(SMEM_BWD <= 232448, "backward shared memory exceeds the per-block limit");

constexpr uint32_t RBF_TERM = TILE_E * KP * 2;   // 16 KB: one 16-bit term of a [128 x 64] tile
constexpr uint32_t ACT_TERM = TILE_E * FP * 2;   // 32 KB: one 16-bit term of a [128 x 128] tile
constexpr uint32_t WAIT_POLLS = 1u << 22;

struct EdgeMeta {          // one 16-byte record per edge of the tile
    int32_t row;
    int32_t col;           // -1: padding or d >= r_c (masked)
    float fc;
    float dfc;
};
// Row summary of one 32-edge chunk, written once per tile by warp votes in
// stage R: first and last row, which edges belong to the first row, and
// whether any third row occurs (then the general segmented path is taken).
struct ChunkInfo {
    int32_t rfirst, rlast;
    uint32_t firstmask;
    int32_t other;
};

// Per-edge records of one tile, stored as arrays so that an epilogue thread
// reads four consecutive edges with one 16-byte shared load.  A masked edge
// (d >= r_c, or d = 0) keeps a valid column index and gets f_c = f_c' = 0, so
// it contributes exactly zero without a branch; padding edges past the end of
// the run get row = INT_MAX, column 0 and f_c = f_c' = 0.
struct TileMeta {
    int32_t row[TILE_E];
    int32_t col[TILE_E];
    float fc[TILE_E];
    float dfc[TILE_E];
    ChunkInfo c[TILE_E / 32];
};
static_assert(sizeof(TileMeta) == TILEMETA_BYTES, "tile metadata layout");

__device__ __forceinline__ void copy_weights(uint8_t* smem, const uint8_t* __restrict__ img)
{
    const uint4* src = reinterpret_cast<const uint4*>(img);
    uint4* dst = reinterpret_cast<uint4*>(smem + SM_W1);
    for (int i = threadIdx.x; i < (int)(LAYER_IMG / 16); i += blockDim.x) dst[i] = __ldg(src + i);
}

// two fp32 values -> packed 16-bit hi pair and lo (residual) pair
template <int FMT>
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo);
template <>
__device__ __forceinline__ void split2<0>(float x0, float x1, uint32_t& hi, uint32_t& lo)
{
    __half2 h = __floats2half2_rn(x0, x1);
    float2 hf = __half22float2(h);
    __half2 l = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<uint32_t*>(&h);
    lo = *reinterpret_cast<uint32_t*>(&l);
}
template <>
__device__ __forceinline__ void split2<1>(float x0, float x1, uint32_t& hi, uint32_t& lo)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    float2 hf = __bfloat1622float2(h);
    __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<uint32_t*>(&h);
    lo = *reinterpret_cast<uint32_t*>(&l);
}

// 8 consecutive fp32 values -> one 16-byte hi store and one 16-byte lo store
template <int FMT>
__device__ __forceinline__ void store8(uint8_t* hi_base, uint8_t* lo_base, uint32_t off, const float* v)
{
    uint32_t h[4], l[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) split2<FMT>(v[2 * q], v[2 * q + 1], h[q], l[q]);
    *reinterpret_cast<uint4*>(hi_base + off) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(lo_base + off) = make_uint4(l[0], l[1], l[2], l[3]);
}

// 32 lanes x 16 columns of TMEM -> 16 registers per thread
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16])
{
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
        : "r"(taddr));
}

// Endpoints of edge (threadIdx.x mod 128) of a tile, loaded one tile ahead so the
// dependent loads (edge -> atom -> position) overlap the previous tile's work.
struct EdgePre {
    int i, j;
    float4 pi, pj;
    int gidx;      // backward: index of the edge in the full list (where s_e is stored)
    float sold;    // backward: s_e accumulated by the later interactions so far
};

template <bool BWD = false>
__device__ __forceinline__ EdgePre prefetch_edge(const MPArgs& a, long long e0, int ne)
{
    EdgePre p;
    p.i = 0;
    p.j = -1;
    p.pi = p.pj = make_float4(0.f, 0.f, 0.f, 0.f);
    p.gidx = 0;
    p.sold = 0.f;
    const int t = threadIdx.x & (TILE_E - 1);
    if (t < ne) {
        p.i = __ldg(a.crow + e0 + t);
        p.j = __ldg(a.ccol + e0 + t);
        p.pi = __ldg(a.pos4 + p.i);
        p.pj = __ldg(a.pos4 + p.j);
        if (BWD && threadIdx.x < TILE_E) {
            p.gidx = __ldg(a.cidx + e0 + t);
            if (a.accumulate_s) p.sold = a.s_edge[p.gidx];
        }
    }
    return p;
}

// Stage R: four threads per edge (one per 16 Gaussians): distance (minimum
// image), cutoff mask, Gaussian expansion (and its d-derivative when BWD)
// written as hi/lo 16-bit K-major B operands.  The derivative operand holds
// (d e_k / d d) / (2 ln 2); the backward epilogue folds the factor back in.
// Gaussian columns past K meet zero weight rows, and masked or padding edges
// have f_c = f_c' = 0, so neither needs a mask here (both stay finite).
template <int FMT, bool BWD>
__device__ __forceinline__ void stage_rbf(const MPArgs& a, uint8_t* smem, TileMeta* tmeta, const EdgePre& ep, int ne)
{
    const int e = threadIdx.x & (TILE_E - 1);
    const int kq = threadIdx.x >> 7;
    float d = 0.f;
    bool valid = false;
    if (e < ne) {
        float3 v;
        d = edge_distance(ep.pi, ep.pj, a.box, v);
        valid = d < a.rc && d > 0.f;
    }
    if (kq == 0) {
        float fc = 0.f, dfc = 0.f;
        if (valid) {
            float sn, cs;
            sincospif(d * a.inv_rc, &sn, &cs);
            fc = 0.5f * (cs + 1.0f);
            dfc = -0.5f * 3.14159265358979f * a.inv_rc * sn;
        }
        const int row = e < ne ? ep.i : 0x7fffffff;
        tmeta->row[e] = row;
        tmeta->col[e] = e < ne ? ep.j : 0;
        tmeta->fc[e] = fc;
        if (BWD) tmeta->dfc[e] = dfc;
        // warp w of this quarter holds edges 32w .. 32w+31: summarise the chunk's rows
        const int lane = threadIdx.x & 31, w = e >> 5;
        const int nv = min(max(ne - 32 * w, 0), 32);
        const int rfirst = __shfl_sync(0xffffffffu, row, 0);
        const int rlast = __shfl_sync(0xffffffffu, row, nv > 0 ? nv - 1 : 0);
        const unsigned fm = __ballot_sync(0xffffffffu, e < ne && row == rfirst);
        const int oth = __any_sync(0xffffffffu, e < ne && row != rfirst && row != rlast);
        if (lane == 0) tmeta->c[w] = ChunkInfo{rfirst, rlast, fm, oth};
    }
    uint8_t* b_hi = smem + SM_X;
    uint8_t* b_lo = b_hi + RBF_TERM;
    uint8_t* p_hi = smem + SM_X + 2 * RBF_TERM;   // derivative tile (backward)
    uint8_t* p_lo = p_hi + RBF_TERM;
    const float dm = d - fmaf((float)(kq * 16), a.dmu, a.mu0);   // d - mu of this thread's first Gaussian
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const int kg = kq * 2 + g;
        float gv[8], dv[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float x = fmaf(-(float)(g * 8 + q), a.dmu, dm);
            const float t = x * a.ngc;
            const float gg = ex2_mufu(t * x);
            gv[q] = gg;
            dv[q] = t * gg;
        }
        const uint32_t off = kmajor_off(e, kg * 8, TILE_E);
        store8<FMT>(b_hi, b_lo, off, gv);
        if (BWD) store8<FMT>(p_hi, p_lo, off, dv);
    }
}

// Issue D (+)= W^T * B over `ksteps` K-steps of 16 with the hi/lo split.
template <int NW>
__device__ __forceinline__ void issue_gemm(uint32_t d_tmem, uint32_t a_base, uint32_t a_term, uint32_t b_base,
                                           uint32_t b_term, int ksteps, uint32_t idesc)
{
    for (int ks = 0; ks < ksteps; ++ks) {
        uint32_t koff = (uint32_t)ks * 2u * (uint32_t)(FP * 16);   // 2 core matrices of 8 along K
        uint64_t a_hi = smem_desc(a_base + koff, FP * 16, 128);
        uint64_t a_lo = smem_desc(a_base + a_term + koff, FP * 16, 128);
        uint64_t b_hi = smem_desc(b_base + koff, TILE_E * 16, 128);
        uint64_t b_lo = smem_desc(b_base + b_term + koff, TILE_E * 16, 128);
        mma_f16(d_tmem, a_hi, b_hi, idesc, ks > 0 ? 1u : 0u);
        if (NW == 2) mma_f16(d_tmem, a_lo, b_hi, idesc, 1u);
        mma_f16(d_tmem, a_hi, b_lo, idesc, 1u);
    }
}

// Wait for the tensor-core commit; returns false (uniformly) on timeout.
__device__ __forceinline__ bool wait_mma(uint64_t* bar, uint32_t& phase, DevMeta* meta)
{
    bool ok = true;
    if ((threadIdx.x >> 5) == 0) ok = mbar_wait_bounded(bar, phase, WAIT_POLLS);   // the others sleep below
    phase ^= 1u;
    int bad = __syncthreads_or(!ok);
    if (bad) {
        if (threadIdx.x == 0) set_flag(meta, SCHNET_FLAG_TIMEOUT);
        return false;
    }
    tc_fence_after();
    return true;
}

// x_j,f (one feature per thread, src_f = x + f) for N consecutive edges starting at e;
// the column indices come four at a time from the tile's column array
template <int N>
__device__ __forceinline__ void gather(const float* __restrict__ src_f, const TileMeta* tm, int e, float (&dst)[N])
{
#pragma unroll
    for (int q = 0; q < N; q += 4) {
        const int4 j = *reinterpret_cast<const int4*>(tm->col + e + q);
        dst[q] = __ldg(src_f + (size_t)j.x * FP);
        dst[q + 1] = __ldg(src_f + (size_t)j.y * FP);
        dst[q + 2] = __ldg(src_f + (size_t)j.z * FP);
        dst[q + 3] = __ldg(src_f + (size_t)j.w * FP);
    }
}

// N per-edge values of the tile's array v starting at edge e (16-byte loads)
template <int N>
__device__ __forceinline__ void load_edges(const float* v, int e, float (&dst)[N])
{
#pragma unroll
    for (int q = 0; q < N; q += 4) {
        const float4 x = *reinterpret_cast<const float4*>(v + e + q);
        dst[q] = x.x;
        dst[q + 1] = x.y;
        dst[q + 2] = x.z;
        dst[q + 3] = x.w;
    }
}

// Segmented sum over the edges of one 32-edge chunk (one feature per thread):
// rows that start and end inside the chunk are written out directly (with
// zeros for edge-less rows between them); the chunk's first row and, when
// different, its last row leave partial sums (pf, pl) for the in-order merge.
struct ChunkSeg {
    int rfirst, lrow;
    float acc, pf;
};

__device__ __forceinline__ void seg_begin(ChunkSeg& c, const TileMeta* tm, int eb)
{
    c.rfirst = tm->row[eb];
    c.lrow = c.rfirst;
    c.acc = 0.f;
    c.pf = 0.f;
}

__device__ __forceinline__ void seg_row(ChunkSeg& c, int row, float* __restrict__ out, int f)
{
    if (row != c.lrow) {
        if (c.lrow == c.rfirst) c.pf = c.acc;
        else out[(size_t)c.lrow * FP + f] = c.acc;
        for (int rr = c.lrow + 1; rr < row; ++rr) out[(size_t)rr * FP + f] = 0.f;
        c.lrow = row;
        c.acc = 0.f;
    }
}

// In-order merge of the four chunks' partials (threads 0..127, feature f).
__device__ __forceinline__ void merge_chunks(const TileMeta* tm, const float* pf, const float* pl, int ne, int f,
                                             float* __restrict__ out, int& cur, float& acc)
{
#pragma unroll 1
    for (int c = 0; c < TILE_E / 32; ++c) {
        const int eb = c * 32;
        if (eb >= ne) break;
        const int last = min(eb + 31, ne - 1);
        const int rfirst = tm->c[c].rfirst, rlast = tm->c[c].rlast;
        (void)last;
        const float v = pf[c * 128 + f];
        if (rfirst == cur) {
            acc += v;
        } else {
            out[(size_t)cur * FP + f] = acc;
            for (int rr = cur + 1; rr < rfirst; ++rr) out[(size_t)rr * FP + f] = 0.f;
            cur = rfirst;
            acc = v;
        }
        if (rlast != rfirst) {
            out[(size_t)cur * FP + f] = acc;
            cur = rlast;
            acc = pl[c * 128 + f];
        }
    }
}

// pairwise sum of N values (fixed order)
template <int N>
__device__ __forceinline__ float tree_sum(float (&v)[N])
{
#pragma unroll
    for (int w = N / 2; w >= 1; w >>= 1)
#pragma unroll
        for (int q = 0; q < w; ++q) v[q] += v[q + w];
    return v[0];
}

// Reduce a chunk's per-edge terms t[q] (edge eb + q) to the first-row and
// last-row partials.  One or two rows: branch-free predicated sums (edge-less
// rows strictly between them are written as zeros).  Three or more rows: the
// serial segmented sum writes the inner rows out.
template <int N>
__device__ __forceinline__ void chunk_partials(const TileMeta* tm, int cidx, int eb, int ne, float (&t)[N],
                                               float* __restrict__ out, int f, float& pf, float& pl)
{
    const ChunkInfo ci = tm->c[cidx];
    if (!ci.other) {
        if (ci.rfirst == ci.rlast) {
            pf = tree_sum<N>(t);
            pl = 0.f;
        } else {
            float u[N];
#pragma unroll
            for (int q = 0; q < N; ++q) {
                const bool first = (ci.firstmask >> q) & 1u;
                u[q] = first ? 0.f : t[q];
                t[q] = first ? t[q] : 0.f;
            }
            pf = tree_sum<N>(t);
            pl = tree_sum<N>(u);
            for (int rr = ci.rfirst + 1; rr < ci.rlast; ++rr) out[(size_t)rr * FP + f] = 0.f;
        }
        return;
    }
    ChunkSeg c{0, 0, 0.f, 0.f};
    seg_begin(c, tm, eb);
#pragma unroll
    for (int q = 0; q < N; ++q) {
        const int e = eb + q;
        if (e >= ne) break;
        seg_row(c, tm->row[e], out, f);
        c.acc += t[q];
    }
    if (c.lrow == c.rfirst) { pf = c.acc; pl = 0.f; } else { pf = c.pf; pl = c.acc; }
}

// forward epilogue 1 for this warp's 32 edges: a = sp2(s1 log2e P + b1 log2e) -> MN-major
// B operand (the base-2 softplus; ssp = ln2 (a - 1), with ln2 and the shift folded
// into the second layer's scale and bias)
template <int FMT>
__device__ __forceinline__ void fwd_e1(uint32_t tP, float s1L, float b1L, uint8_t* smem, int cg, int f)
{
    float r[32];
    tmem_ld32(tP, r);
    tmem_ld_wait();
#pragma unroll
    for (int q = 0; q < 32; ++q) r[q] = sp2(fmaf(s1L, r[q], b1L));
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const uint32_t off = mnmajor_off(cg * 32 + g * 8, f, TILE_E);
        store8<FMT>(smem + SM_FWD_A, smem + SM_FWD_A + ACT_TERM, off, r + g * 8);
    }
}

// forward epilogue 2 for this warp's chunk: W = f_c (s2 ln2 Q + b2s), terms h_j W, chunk partials
__device__ __forceinline__ void fwd_e2(uint32_t tQ, const TileMeta* tm, int cg, int ne, float s2L, float b2s,
                                       const float (&hv)[32], float* __restrict__ out, int f, float& pf, float& pl)
{
    float r[32];
    tmem_ld32(tQ, r);
    tmem_ld_wait();
    const int eb = cg * 32;
    pf = pl = 0.f;
    if (eb >= ne) return;
    float fc[32];
    load_edges<32>(tm->fc, eb, fc);
#pragma unroll
    for (int q = 0; q < 32; ++q) r[q] = fc[q] * fmaf(s2L, r[q], b2s) * hv[q];
    chunk_partials<32>(tm, cg, eb, ne, r, out, f, pf, pl);
}

// ---------------------------------------------------------------------------
// forward: m_i = sum_j h_j (.) W(d_ij)
// ---------------------------------------------------------------------------
template <int FMT, int NW>
__global__ void __launch_bounds__(NT, 1) k_cfconv_fwd(MPArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    auto tmb = [&](int t) { return reinterpret_cast<TileMeta*>(smem + SM_META_FWD + (t & 1) * TILEMETA_BYTES); };
    float* pf_s = reinterpret_cast<float*>(smem + SM_META_FWD + 2 * TILEMETA_BYTES);
    float* pl_s = pf_s + 4 * 128;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + SM_META_FWD + 2 * TILEMETA_BYTES + PART_BYTES);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + SM_META_FWD + 2 * TILEMETA_BYTES + PART_BYTES + 8);

    if (a.meta->n_edges > a.cap) return;
    const int r0 = a.part[blockIdx.x], r1 = a.part[blockIdx.x + 1];
    if (r0 >= r1) return;
    const long long e0 = a.row_ptr[r0], e1 = e0 + a.ccount[blockIdx.x];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qd = warp & 3, cg = warp >> 2;        // TMEM lane quadrant, 32-edge column chunk
    const int f = qd * 32 + lane;                   // this thread's output feature

    if (warp == 0) {
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    copy_weights(smem, a.img);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const uint32_t tP = tmem + lane_off + cg * 32, tQ = tmem + 128 + lane_off + cg * 32;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t id = idesc_f16(128, TILE_E, FMT, 0);
    const uint32_t id_mn = idesc_f16(128, TILE_E, FMT, 1);

    const float s1L = a.s1[f] * LOG2EF, b1L = a.b1[f] * LOG2EF;
    const float s2L = a.s2[f] * LN2F, b2s = a.b2s[f];
    const float* h_f = a.h + f;
    int cur = r0;          // carried row and partial sum (threads 0..127, feature = threadIdx.x)
    float acc = 0.f;
    uint32_t phase = 0;
    bool ok = true;
    const int ntiles = (int)((e1 - e0 + TILE_E - 1) / TILE_E);
    auto tile_ne = [&](int t) { return (int)min((long long)TILE_E, e1 - e0 - (long long)t * TILE_E); };

    // Software pipeline: tile t's GEMM2 runs while stage R of tile t+1 fills the
    // Gaussian operand; tile t's epilogue 2 runs while GEMM1 of tile t+1 runs.
    if (ntiles > 0) {
        EdgePre ep = prefetch_edge(a, e0, tile_ne(0));
        stage_rbf<FMT, false>(a, smem, tmb(0), ep, tile_ne(0));
        if (ntiles > 1) ep = prefetch_edge(a, e0 + TILE_E, tile_ne(1));
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            issue_gemm<NW>(tmem, sbase + SM_W1, (uint32_t)W1_IMG, sbase + SM_X, RBF_TERM, KP / 16, id);
            mma_commit(bar);
        }
        ok = wait_mma(bar, phase, a.meta);
        if (ok) {
            fwd_e1<FMT>(tP, s1L, b1L, smem, cg, f);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            if (threadIdx.x == 0) {
                tc_fence_after();
                issue_gemm<NW>(tmem + 128, sbase + SM_W2, (uint32_t)W2_IMG, sbase + SM_FWD_A, ACT_TERM, FP / 16,
                               id_mn);
                mma_commit(bar);
            }
        }
        for (int t = 0; t < ntiles && ok; ++t) {
            const int ne = tile_ne(t);
            const bool next = t + 1 < ntiles;
            TileMeta* tm = tmb(t);
            // (GEMM2 of tile t in flight) Gaussians of the next tile, then this chunk's h_j rows
            if (next) {
                stage_rbf<FMT, false>(a, smem, tmb(t + 1), ep, tile_ne(t + 1));
                fence_proxy_async_smem();
                if (t + 2 < ntiles) ep = prefetch_edge(a, e0 + (long long)(t + 2) * TILE_E, tile_ne(t + 2));
            }
            float hv[32];
            gather<32>(h_f, tm, cg * 32, hv);
            if (!(ok = wait_mma(bar, phase, a.meta))) break;      // GEMM2(t) done; next tile's operand ready
            if (next && threadIdx.x == 0) {
                issue_gemm<NW>(tmem, sbase + SM_W1, (uint32_t)W1_IMG, sbase + SM_X, RBF_TERM, KP / 16, id);
                mma_commit(bar);
            }
            // (GEMM1 of tile t+1 in flight) epilogue 2 and the in-order merge of tile t
            float pf, pl;
            fwd_e2(tQ, tm, cg, ne, s2L, b2s, hv, a.out, f, pf, pl);
            pf_s[cg * 128 + f] = pf;
            pl_s[cg * 128 + f] = pl;
            __syncthreads();
            if (threadIdx.x < 128) merge_chunks(tm, pf_s, pl_s, ne, threadIdx.x, a.out, cur, acc);
            if (next) {
                if (!(ok = wait_mma(bar, phase, a.meta))) break;  // GEMM1(t+1) done
                fwd_e1<FMT>(tP, s1L, b1L, smem, cg, f);
                fence_proxy_async_smem();
                tc_fence_before();
                __syncthreads();
                if (threadIdx.x == 0) {
                    tc_fence_after();
                    issue_gemm<NW>(tmem + 128, sbase + SM_W2, (uint32_t)W2_IMG, sbase + SM_FWD_A, ACT_TERM,
                                   FP / 16, id_mn);
                    mma_commit(bar);
                }
            } else {
                __syncthreads();
            }
        }
    }

    if (ok) {
        if (threadIdx.x < 128) {
            a.out[(size_t)cur * FP + threadIdx.x] = acc;
            for (int rr = cur + 1; rr < r1; ++rr) a.out[(size_t)rr * FP + threadIdx.x] = 0.f;
        }
    } else {
        // drain: give in-flight MMAs a bounded chance to retire before freeing TMEM
        mbar_wait_bounded(bar, phase, WAIT_POLLS);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ---------------------------------------------------------------------------
// backward: dh_i = sum_j u_j (.) W_ij ;  s_e = sum_f W'_e,f u_i,f h_j,f
// ---------------------------------------------------------------------------
// backward epilogue 1 for this warp's 32 edges: a = sp2(p), b = ssp'(x) dx/dd, with
// p = x log2e = s1 log2e P + b1 log2e and dx/dd = s1 2ln2 P' (P' from the scaled
// Gaussian-derivative operand).  ssp'(x) = 1 / (1 + e^-x) shares 2^-|p| with sp2.
template <int FMT>
__device__ __forceinline__ void bwd_e1(uint32_t tP, uint32_t tPd, float s1L, float b1L, float s1d, uint8_t* smem,
                                       uint32_t col0, int f)
{
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float r[16], rd[16];
        tmem_ld16(tP + hh * 16, r);
        tmem_ld16(tPd + hh * 16, rd);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const float p = fmaf(s1L, r[q], b1L);
            const float t = ex2_mufu(-fabsf(p));
            const float y = 1.0f + t;
            const float inv = rcp_mufu(y);
            const float sg = p >= 0.0f ? inv : t * inv;       // logistic(x)
            r[q] = fmaxf(p, 0.0f) + lg2_mufu(y);
            rd[q] = sg * (s1d * rd[q]);
        }
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            const uint32_t off = mnmajor_off(col0 + hh * 16 + g * 8, f, TILE_E);
            store8<FMT>(smem + SM_X, smem + SM_X + ACT_TERM, off, r + g * 8);
            store8<FMT>(smem + SM_BWD_Y, smem + SM_BWD_Y + ACT_TERM, off, rd + g * 8);
        }
    }
}

template <int FMT, int NW>
__global__ void __launch_bounds__(NT, 1) k_cfconv_bwd(MPArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    TileMeta* tm = reinterpret_cast<TileMeta*>(smem + SM_META_BWD);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + SM_META_BWD + TILEMETA_BYTES);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + SM_META_BWD + TILEMETA_BYTES + 8);
    // after GEMM2 the ssp'(p)p' tile is dead: its space holds the partial sums and,
    // behind them, the next tile's metadata until the merge has finished with tm
    float* pf_s = reinterpret_cast<float*>(smem + SM_BWD_Y);
    float* pl_s = pf_s + 4 * 128;
    float* ps_s = pl_s + 4 * 128;   // [quadrant][edge] per-edge partial of s_e
    TileMeta* tm_next = reinterpret_cast<TileMeta*>(smem + SM_BWD_Y + 8192);

    if (a.meta->n_edges > a.cap) return;
    const int r0 = a.part[blockIdx.x], r1 = a.part[blockIdx.x + 1];
    if (r0 >= r1) return;
    const long long e0 = a.row_ptr[r0], e1 = e0 + a.ccount[blockIdx.x];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qd = warp & 3, cg = warp >> 2;
    const int f = qd * 32 + lane;

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    copy_weights(smem, a.img);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const uint32_t col0 = cg * 32;
    const uint32_t tP = tmem + lane_off + col0, tPd = tmem + 128 + lane_off + col0;
    const uint32_t tQ = tmem + 256 + lane_off + col0, tQd = tmem + 384 + lane_off + col0;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t id = idesc_f16(128, TILE_E, FMT, 0);
    const uint32_t id_mn = idesc_f16(128, TILE_E, FMT, 1);

    const float s1L = a.s1[f] * LOG2EF, b1L = a.b1[f] * LOG2EF, s1d = a.s1[f] * (2.0f * LN2F);
    const float s2 = a.s2[f], s2L = a.s2[f] * LN2F, b2s = a.b2s[f];
    const float* h_f = a.h + f;
    const float* u_f = a.u + f;
    int cur = r0;
    float acc = 0.f;
    uint32_t phase = 0;
    bool ok = true;
    const int ntiles = (int)((e1 - e0 + TILE_E - 1) / TILE_E);
    auto tile_ne = [&](int t) { return (int)min((long long)TILE_E, e1 - e0 - (long long)t * TILE_E); };
    int cur_g = 0, nxt_g = 0;           // threads < 128: s_e slot of edge threadIdx.x (this / next tile)
    float cur_so = 0.f, nxt_so = 0.f;

    // Software pipeline: epilogue 2 of tile t runs while GEMM1 of tile t+1 runs.
    if (ntiles > 0) {
        EdgePre ep = prefetch_edge<true>(a, e0, tile_ne(0));
        stage_rbf<FMT, true>(a, smem, tm, ep, tile_ne(0));
        cur_g = ep.gidx;
        cur_so = ep.sold;
        if (ntiles > 1) ep = prefetch_edge<true>(a, e0 + TILE_E, tile_ne(1));
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            issue_gemm<NW>(tmem, sbase + SM_W1, (uint32_t)W1_IMG, sbase + SM_X, RBF_TERM, KP / 16, id);
            issue_gemm<NW>(tmem + 128, sbase + SM_W1, (uint32_t)W1_IMG, sbase + SM_X + 2 * RBF_TERM, RBF_TERM,
                           KP / 16, id);
            mma_commit(bar);
        }
        ok = wait_mma(bar, phase, a.meta);
        if (ok) {
            bwd_e1<FMT>(tP, tPd, s1L, b1L, s1d, smem, col0, f);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            if (threadIdx.x == 0) {
                tc_fence_after();
                issue_gemm<NW>(tmem + 256, sbase + SM_W2, (uint32_t)W2_IMG, sbase + SM_X, ACT_TERM, FP / 16, id_mn);
                issue_gemm<NW>(tmem + 384, sbase + SM_W2, (uint32_t)W2_IMG, sbase + SM_BWD_Y, ACT_TERM, FP / 16,
                               id_mn);
                mma_commit(bar);
            }
        }
        for (int t = 0; t < ntiles && ok; ++t) {
            const int ne = tile_ne(t);
            const bool next = t + 1 < ntiles;
            const long long t0 = e0 + (long long)t * TILE_E;
            const int eb = (int)col0;
            float uv[16], hv[16];
            gather<16>(u_f, tm, eb, uv);
            gather<16>(h_f, tm, eb, hv);
            if (!(ok = wait_mma(bar, phase, a.meta))) break;            // GEMM2(t) done
            if (next) {
                // Gaussians of the next tile into the (now dead) ssp(p) region; its metadata is staged
                stage_rbf<FMT, true>(a, smem, tm_next, ep, tile_ne(t + 1));
                nxt_g = ep.gidx;
                nxt_so = ep.sold;
                if (t + 2 < ntiles) ep = prefetch_edge<true>(a, e0 + (long long)(t + 2) * TILE_E, tile_ne(t + 2));
                fence_proxy_async_smem();
                tc_fence_before();
                __syncthreads();
                if (threadIdx.x == 0) {
                    tc_fence_after();
                    issue_gemm<NW>(tmem, sbase + SM_W1, (uint32_t)W1_IMG, sbase + SM_X, RBF_TERM, KP / 16, id);
                    issue_gemm<NW>(tmem + 128, sbase + SM_W1, (uint32_t)W1_IMG, sbase + SM_X + 2 * RBF_TERM,
                                   RBF_TERM, KP / 16, id);
                    mma_commit(bar);
                }
            }
            // epilogue 2: W = f_c z, W' = f_c' z + f_c z'  (z = s2 ln2 Q + b2s, z' = s2 Q')
            {
                const bool active = eb < ne;
                const ChunkInfo ci = tm->c[cg];
                // 1: one row in the chunk; 2: two rows (the first a prefix); 3: the general
                // serial segmented sum with a row change test per edge
                const int kind = !active ? 0 : ci.other ? 3 : (ci.rfirst == ci.rlast ? 1 : 2);
                float pf = 0.f, pl = 0.f;
                if (kind != 0) {
                    const float u_first = __ldg(u_f + (size_t)ci.rfirst * FP);
                    const float u_last = __ldg(u_f + (size_t)ci.rlast * FP);
                    float sf = 0.f, sl = 0.f;
                    ChunkSeg c{0, 0, 0.f, 0.f};
                    if (kind == 3) seg_begin(c, tm, eb);
                    float u_row = u_first;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        if (hh == 1) {
                            gather<16>(u_f, tm, eb + 16, uv);
                            gather<16>(h_f, tm, eb + 16, hv);
                        }
                        float r[16], rd[16];
                        tmem_ld16(tQ + hh * 16, r);
                        tmem_ld16(tQd + hh * 16, rd);
                        tmem_ld_wait();
                        const float* fcp = tm->fc + eb + hh * 16;
                        const float* dfcp = tm->dfc + eb + hh * 16;
                        if (kind == 1) {
#pragma unroll
                            for (int g = 0; g < 16; g += 4) {
                                float fc[4], dfc[4];
                                load_edges<4>(fcp, g, fc);
                                load_edges<4>(dfcp, g, dfc);
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const int q = g + i;
                                    const float z = fmaf(s2L, r[q], b2s);
                                    sf = fmaf(fc[i] * z, uv[q], sf);
                                    const float wd = fmaf(dfc[i], z, fc[i] * (s2 * rd[q]));
                                    rd[q] = wd * (u_first * hv[q]);
                                }
                            }
                        } else if (kind == 2) {
#pragma unroll
                            for (int g = 0; g < 16; g += 4) {
                                float fc[4], dfc[4];
                                load_edges<4>(fcp, g, fc);
                                load_edges<4>(dfcp, g, dfc);
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const int q = g + i;
                                    const float z = fmaf(s2L, r[q], b2s);
                                    const float dt = fc[i] * z * uv[q];
                                    const bool first = (ci.firstmask >> (hh * 16 + q)) & 1u;
                                    sf += first ? dt : 0.f;
                                    sl += first ? 0.f : dt;
                                    const float wd = fmaf(dfc[i], z, fc[i] * (s2 * rd[q]));
                                    rd[q] = wd * ((first ? u_first : u_last) * hv[q]);
                                }
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < 16; ++q) {
                                const int e = eb + hh * 16 + q;
                                float tval = 0.f;
                                if (e < ne) {
                                    const int row = tm->row[e];
                                    if (row != c.lrow) {
                                        seg_row(c, row, a.out, f);
                                        u_row = __ldg(u_f + (size_t)row * FP);
                                    }
                                    const float fcq = fcp[q], dfcq = dfcp[q];
                                    const float z = fmaf(s2L, r[q], b2s);
                                    const float wd = fmaf(dfcq, z, fcq * (s2 * rd[q]));
                                    c.acc = fmaf(fcq * z, uv[q], c.acc);
                                    tval = wd * (u_row * hv[q]);
                                }
                                rd[q] = tval;
                            }
                        }
                        // transpose-reduce the 16 per-edge values over the warp's 32 features:
                        // afterwards lanes 2k and 2k+1 hold the sum for edge k of this half
#pragma unroll
                        for (int sh = 16; sh >= 2; sh >>= 1) {
                            const bool upper = (lane & sh) != 0;
#pragma unroll
                            for (int k = 0; k < sh / 2; ++k) {
                                float send = upper ? rd[k] : rd[k + sh / 2];
                                float keep = upper ? rd[k + sh / 2] : rd[k];
                                rd[k] = keep + __shfl_xor_sync(0xffffffffu, send, sh);
                            }
                        }
                        rd[0] += __shfl_xor_sync(0xffffffffu, rd[0], 1);
                        if ((lane & 1) == 0) ps_s[qd * TILE_E + eb + hh * 16 + (lane >> 1)] = rd[0];
                    }
                    if (kind == 1) {
                        pf = sf;
                    } else if (kind == 2) {
                        pf = sf;
                        pl = sl;
                        for (int rr = ci.rfirst + 1; rr < ci.rlast; ++rr) a.out[(size_t)rr * FP + f] = 0.f;
                    } else if (c.lrow == c.rfirst) {
                        pf = c.acc;
                    } else {
                        pf = c.pf;
                        pl = c.acc;
                    }
                }
                pf_s[cg * 128 + f] = pf;
                pl_s[cg * 128 + f] = pl;
            }
            __syncthreads();
            if (threadIdx.x < 128) {
                merge_chunks(tm, pf_s, pl_s, ne, threadIdx.x, a.out, cur, acc);
                if ((int)threadIdx.x < ne) {
                    const int q = threadIdx.x;
                    const float sv = ps_s[q] + ps_s[TILE_E + q] + ps_s[2 * TILE_E + q] + ps_s[3 * TILE_E + q];
                    a.s_edge[cur_g] = a.accumulate_s ? cur_so + sv : sv;
                }
            }
            if (next) {
                __syncthreads();                                        // merge done with tm
                for (int i = threadIdx.x; i < (int)(sizeof(TileMeta) / 4); i += NT)
                    reinterpret_cast<uint32_t*>(tm)[i] = reinterpret_cast<const uint32_t*>(tm_next)[i];
                cur_g = nxt_g;
                cur_so = nxt_so;
                if (!(ok = wait_mma(bar, phase, a.meta))) break;        // GEMM1(t+1) done
                bwd_e1<FMT>(tP, tPd, s1L, b1L, s1d, smem, col0, f);
                fence_proxy_async_smem();
                tc_fence_before();
                __syncthreads();
                if (threadIdx.x == 0) {
                    tc_fence_after();
                    issue_gemm<NW>(tmem + 256, sbase + SM_W2, (uint32_t)W2_IMG, sbase + SM_X, ACT_TERM, FP / 16,
                                   id_mn);
                    issue_gemm<NW>(tmem + 384, sbase + SM_W2, (uint32_t)W2_IMG, sbase + SM_BWD_Y, ACT_TERM, FP / 16,
                                   id_mn);
                    mma_commit(bar);
                }
            } else {
                __syncthreads();
            }
        }
    }

    if (ok) {
        if (threadIdx.x < 128) {
            a.out[(size_t)cur * FP + threadIdx.x] = acc;
            for (int rr = cur + 1; rr < r1; ++rr) a.out[(size_t)rr * FP + threadIdx.x] = 0.f;
        }
    } else {
        mbar_wait_bounded(bar, phase, WAIT_POLLS);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// cutoff masking: per CTA row range, the listed edges with d < r_c, in order
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_compact(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ part,
                                                  const int32_t* __restrict__ erow, const int32_t* __restrict__ col,
                                                  const float4* __restrict__ pos4, Box box, float rc, long long cap,
                                                  const DevMeta* meta, int32_t* __restrict__ crow,
                                                  int32_t* __restrict__ ccol, int32_t* __restrict__ cidx,
                                                  int32_t* __restrict__ ccount)
{
    __shared__ int wcount[32];
    __shared__ int total_s;
    const int c = blockIdx.x;
    const int r0 = part[c], r1 = part[c + 1];
    if (meta->n_edges > cap || r0 >= r1) {
        if (threadIdx.x == 0) ccount[c] = 0;
        return;
    }
    const long long e0 = row_ptr[r0], e1 = row_ptr[r1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long base = e0;
    for (long long eb = e0; eb < e1; eb += blockDim.x) {
        const long long e = eb + threadIdx.x;
        bool valid = false;
        int i = 0, j = 0;
        if (e < e1) {
            i = erow[e];
            j = col[e];
            float3 v;
            const float d = edge_distance(pos4[i], pos4[j], box, v);
            valid = d < rc && d > 0.f;
        }
        const unsigned mask = __ballot_sync(0xffffffffu, valid);
        if (lane == 0) wcount[warp] = __popc(mask);
        __syncthreads();
        if (warp == 0) {
            int v = wcount[lane];
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            wcount[lane] = incl - v;
            if (lane == 31) total_s = incl;
        }
        __syncthreads();
        if (valid) {
            const long long k = base + wcount[warp] + __popc(mask & ((1u << lane) - 1u));
            crow[k] = i;
            ccol[k] = j;
            cidx[k] = (int32_t)e;
        }
        base += total_s;
        __syncthreads();
    }
    if (threadIdx.x == 0) ccount[c] = (int32_t)(base - e0);
}

cudaError_t launch_compact(schnet_ctx* c)
{
    Workspace& w = c->ws;
    k_compact<<<c->ncta, 1024, 0, c->s>>>(w.row_ptr, w.part, w.erow, w.col, w.pos4, c->box, c->cfg.cutoff, c->cap,
                                          w.meta, w.crow, w.ccol, w.cidx, w.ccount);
    c->launches += 1;
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
static MPArgs make_args(schnet_ctx* c, int layer)
{
    Workspace& w = c->ws;
    MPArgs a;
    a.pos4 = w.pos4;
    a.crow = w.crow;
    a.ccol = w.ccol;
    a.cidx = w.cidx;
    a.ccount = w.ccount;
    a.row_ptr = w.row_ptr;
    a.part = w.part;
    a.meta = w.meta;
    a.cap = c->cap;
    a.box = c->box;
    a.rc = c->cfg.cutoff;
    a.inv_rc = 1.0f / c->cfg.cutoff;
    a.mu0 = c->mu0;
    a.dmu = c->dmu;
    a.ngc = (float)(-1.4426950408889634 / (2.0 * (double)c->cfg.rbf_sigma * (double)c->cfg.rbf_sigma));
    a.img = w.img + (size_t)layer * LAYER_IMG;
    a.s1 = w.s1 + layer * FP;
    a.s2 = w.s2 + layer * FP;
    a.b1 = w.b1 + layer * FP;
    a.b2s = w.b2s + layer * FP;
    a.h = w.h + (size_t)layer * c->N * FP;
    a.u = w.m;
    a.out = nullptr;
    a.s_edge = w.s_edge;
    a.accumulate_s = 0;
    return a;
}

template <int FMT, int NW>
static cudaError_t set_attrs()
{
    cudaError_t e = cudaFuncSetAttribute(k_cfconv_fwd<FMT, NW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_FWD);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(k_cfconv_bwd<FMT, NW>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BWD);
}

cudaError_t cfconv_init_attributes()
{
    cudaError_t e;
    if ((e = set_attrs<0, 2>()) != cudaSuccess) return e;
    if ((e = set_attrs<0, 1>()) != cudaSuccess) return e;
    return set_attrs<1, 1>();
}

cudaError_t launch_cfconv_fwd(schnet_ctx* c, int layer)
{
    MPArgs a = make_args(c, layer);
    a.out = c->ws.m;
    if (c->weight_fmt == 0 && c->n_wterms == 2)
        k_cfconv_fwd<0, 2><<<c->ncta, NT, SMEM_FWD, c->s>>>(a);
    else if (c->weight_fmt == 0)
        k_cfconv_fwd<0, 1><<<c->ncta, NT, SMEM_FWD, c->s>>>(a);
    else
        k_cfconv_fwd<1, 1><<<c->ncta, NT, SMEM_FWD, c->s>>>(a);
    c->launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_cfconv_bwd(schnet_ctx* c, int layer, int accumulate_s)
{
    MPArgs a = make_args(c, layer);
    a.out = c->ws.dh;
    a.accumulate_s = accumulate_s;
    if (c->weight_fmt == 0 && c->n_wterms == 2)
        k_cfconv_bwd<0, 2><<<c->ncta, NT, SMEM_BWD, c->s>>>(a);
    else if (c->weight_fmt == 0)
        k_cfconv_bwd<0, 1><<<c->ncta, NT, SMEM_BWD, c->s>>>(a);
    else
        k_cfconv_bwd<1, 1><<<c->ncta, NT, SMEM_BWD, c->s>>>(a);
    c->launches += 1;
    return cudaGetLastError();
}

}  // namespace schnet
