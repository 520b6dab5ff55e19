// Fused continuous-filter convolution on the sm_100a tensor cores.
//
// One kernel per interaction and direction does, for tiles of a CTA's contiguous
// CSR rows (forward: 128 edges; backward: 64 edges, whose derivative rows fill
// the other half of the GEMM's N = 128):
//   flash radial basis  (FlashSchNet paper-curation summary, How): Gaussian
//     expansion and cosine envelope of the edge's distance (stored by the
//     cutoff-masking pass) computed once per edge into shared memory, never to
//     HBM;
//   filter network      (How, quantization item; contraction on tensor cores):
//     W(d) = f_c(d) (ssp(e W1 + b1) W2 + b2) as two chained tcgen05 GEMMs with
//     TMEM accumulators; channel-wise scaled 16-bit operands, hi/lo split of
//     the activations (and of fp32-stored weights) with fp32 accumulation;
//   flash message passing + flash aggregation (How): cutoff masking, gather of
//     h_j, filter product and the CSR segment sum m_i = sum_j h_j (.) W_ij,
//     accumulated in registers, no atomics, no edge tensor in HBM.
// The backward kernel visits each unordered pair once (the half list, exploiting
// W_ij = W_ji), recomputes W and its distance derivative W' by forward-mode
// tangents, and produces the pair's derivative sum_f W'_f (u_i h_j + u_j h_i)
// and the half list's terms of dE/dh_i = sum_j W_ij (.) u_j; the forward kernel
// over the complementary list adds the other terms.
//
// Tile orientation: the GEMMs are computed transposed, D[f][e] = W^T[f][k] B[e][k],
// so TMEM lane = output feature and TMEM column = edge.  Each epilogue thread
// then owns one feature of every edge in the tile, the per-row reduction is a
// running sum in one register, and the h_j gathers are 128-byte coalesced rows.
// The weights (A) sit in tensor memory; only the edge operands (B) are read
// from shared memory.  Every MMA has N = 128: a tcgen05 MMA of N = 64 costs
// 70 % of the time of one of N = 128 for half the work, so the backward kernel
// stacks each edge's value and derivative operands into one B tile instead of
// issuing two N = 64 GEMMs.
//
// Ping-pong: the CTA's 16 warps form two math groups of 8 warps.  Group g takes
// tiles g, g+2, g+4, ... of the CTA's edge run, each with its own TMEM columns,
// shared-memory operand buffers, named barrier and MMA mbarrier; the two groups
// share only the filter weights (read-only) and the tensor core.  While one
// group waits for its GEMMs or its gathers, the other issues.  The CSR segment
// sums cross tile boundaries through a carry (current row, partial sum per
// feature) handed from tile to tile in order by an mbarrier token.  Group 1
// starts once group 0's first GEMM1 has completed.
//
// Warp roles inside a group: warp 0 issues GEMM2 (an issuing thread blocks while
// the tensor core's queue is full) and so takes no part in stage R (the
// Gaussians of tile t+2, run by warps 1-7 under GEMM2); warp 4 issues the next
// GEMM1 while warps 0-3 merge the segment sums.  In the backward kernel an
// mbarrier token also orders the two groups' epilogues 1 in tile order, which
// keeps their MUFU-bound phases from overlapping and the groups out of step.
#include "internal.h"

namespace schnet {

struct MPArgs {
    const float* cdist;      // distance of each compacted edge (minimum image), from the masking pass
    const int32_t* crow;     // compacted edges (d < r_c) of each CTA's rows: row, column,
    const int32_t* ccol;     //   and index in the full list; CTA c's run starts at
    const int32_t* cidx;     //   row_ptr[part[c]] and holds ccount[c] edges
    const int32_t* ccount;
    const int32_t* row_ptr;
    const int32_t* part;
    DevMeta* meta;
    long long cap;
    float rc, inv_rc;
    float mu0, dmu;       // Gaussian centres mu_k = mu0 + k dmu
    float ngc;            // -log2(e) / (2 sigma^2): e_k = 2^(ngc (d - mu_k)^2)
    int K;                // Gaussians (columns K .. KP-1 are padding)
    const uint8_t* img;   // this layer's packed W1^T / W2^T images
    const float *s1, *s2, *b1;  // this layer's channel scales and first-layer bias [FP]
    const float* b2;      // this layer's second-layer bias [FP]
    const float* h;       // [N][FP]   gathered per edge: h (forward), u = dE/dm (dE/dh launch), h (pairs)
    const float* u;       // [N][FP]   u = dE/dm (pair kernel)
    float* out;           // [N][FP]   m, or dE/dh (forward kernel)
    float* s_edge;        // [cap]     pair derivatives on their owning edges (pair kernel)
    int accumulate_s;     //           add to the later interactions' values
};

constexpr int NT = 512;                  // threads per CTA: two math groups of 8 warps
constexpr int GT = 256;                  // threads per math group
constexpr int MN = 128;                  // GEMM N of every MMA
constexpr int TE_F = 128;                // forward: edges per tile
constexpr int TE_B = 64;                 // backward: edges per tile (B rows 64..127 hold their derivatives)

// TMEM columns (512 allocated): each group's accumulator (P, then Q over it), and
// the filter weights as the MMAs' A operand, one row (output channel) per lane,
// two 16-bit K elements per 32-bit column.
constexpr uint32_t TM_ACC = 128;         // group g: columns g*128 .. g*128+127
constexpr uint32_t TM_W1H = 256, TM_W1L = 288, TM_W2H = 320, TM_W2L = 384;

// shared-memory map (bytes)
constexpr uint32_t RBF_TERM = MN * KP * 2;   // 16 KB: one 16-bit term of a [128 x 64] GEMM1 B tile
constexpr uint32_t ACT_TERM = MN * FP * 2;   // 32 KB: one 16-bit term of a [128 x 128] GEMM2 B tile
constexpr uint32_t SM_RBF = 0;               // group g: GEMM1 B operand hi/lo at g * 32 KB
constexpr uint32_t SM_ACT = 65536;           // group g: GEMM2 B operand hi/lo at 64 KB + g * 64 KB;
                                             //   after GEMM2 it holds the epilogue's partial sums
constexpr uint32_t CARRY_BYTES = FP * 4 + 16;  // carried partial per feature + row (x2)
constexpr uint32_t BAR_BYTES = 64;
constexpr uint32_t WAIT_POLLS = 1u << 22;

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
// the run get column 0 and f_c = f_c' = 0.  Row indices stay in global memory
// (only chunks that hold three or more rows read them).
template <int TE, bool BWD>
struct TileMeta {
    int32_t col[TE];
    float fc[TE];
    float dfc[BWD ? TE : 4];
    float d[TE];                 // distance (stage R's Gaussian units read it)
    ChunkInfo c[TE / 32];
};

// metadata: [group][buffer] (double-buffered per group: stage R of tile t+2
// fills one while the epilogue and merge of tile t read the other)
template <int TE, bool BWD> constexpr uint32_t sm_meta() { return SM_ACT + 2 * 2 * ACT_TERM; }
template <int TE, bool BWD> constexpr uint32_t sm_carry() { return sm_meta<TE, BWD>() + 4 * sizeof(TileMeta<TE, BWD>); }
template <int TE, bool BWD> constexpr uint32_t sm_bar() { return sm_carry<TE, BWD>() + CARRY_BYTES; }
template <int TE, bool BWD> constexpr uint32_t smem_bytes() { return sm_bar<TE, BWD>() + BAR_BYTES; }
// barrier block: [0] group 0 MMA commits, [1] group 1 MMA commits, [2] merge token,
// [3] group 1 start, [4] epilogue-1 token (u64 each); then the TMEM base (u32), each
// group's MMA phase to drain on an error exit (u32 x2) and each group's "commit
// outstanding" flag (u32 x2)
static_assert(smem_bytes<TE_F, false>() <= 232448, "forward shared memory exceeds the per-block limit");
static_assert(smem_bytes<TE_B, true>() <= 232448, "backward shared memory exceeds the per-block limit");
static_assert(sizeof(TileMeta<TE_F, false>) % 16 == 0 && sizeof(TileMeta<TE_B, true>) % 16 == 0, "meta alignment");
static_assert(2 * RBF_TERM * 2 <= SM_ACT, "GEMM1 operands");

// Segment-sum state carried from one tile to the next (in tile order, across
// the two groups): the open row and its partial sum per feature.  The row is
// double-buffered by tile parity, so a slow reader of tile t-1's row never
// races the writer of tile t's.
struct Carry {
    float acc[FP];
    int32_t cur[2];
    int32_t pad[2];
};
static_assert(sizeof(Carry) == CARRY_BYTES, "carry layout");

// named barrier of math group g (ids 1 and 2; id 0 is __syncthreads)
__device__ __forceinline__ void group_sync(int g)
{
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "n"(GT) : "memory");
}

// OR of a predicate over the NTH threads that meet at named barrier id
template <int NTH>
__device__ __forceinline__ bool bar_or(int id, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "n"(NTH)
        : "memory");
    return r != 0;
}

// OR of a predicate over math group g (a barrier of the group's 256 threads, ids 1, 2)
__device__ __forceinline__ bool group_or(int g, bool v) { return bar_or<GT>(1 + g, v); }

// OR of a predicate over the merging warps 0-3 of math group g (ids 3, 4): the
// merge waits for no other warp of its group, in particular not for the one
// issuing the next tile's GEMM1
__device__ __forceinline__ bool merge_or(int g, bool v) { return bar_or<128>(3 + g, v); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Endpoints of edge (group thread mod TE) of a tile, loaded a tile ahead so the
// dependent loads (edge -> atom -> position) overlap the previous tile's work.
struct EdgePre {
    int i, j;
    float d;       // the edge's distance, computed once per step by the masking pass
    int gidx;      // backward: index of the edge in the full list (where s_e is stored)
    float sold;    // backward: s_e accumulated by the later interactions so far
};

template <int TE, bool BWD>
__device__ __forceinline__ EdgePre prefetch_edge(const MPArgs& a, long long e0, int ne, int t)
{
    EdgePre p;
    p.i = 0;
    p.j = -1;
    p.d = 0.f;
    p.gidx = 0;
    p.sold = 0.f;
    if (t >= 0 && t < ne) {
        p.i = __ldg(a.crow + e0 + t);
        p.j = __ldg(a.ccol + e0 + t);
        p.d = __ldg(a.cdist + e0 + t);
        if (BWD) {
            p.gidx = __ldg(a.cidx + e0 + t);
            if (a.accumulate_s) p.sold = a.s_edge[p.gidx];
        }
    }
    return p;
}

// Stage R, by the group's warps 1-7 (worker w = group thread - 32): warp 0 issues
// GEMM2 meanwhile, and an issuing thread blocks while the tensor core's queue is
// full, so warp 0 does no stage-R work.  Workers w < TE take edge w (its endpoints
// and distance prefetched a tile ahead): cutoff envelope f_c (and f_c'), column
// and distance into the tile's record, and a row summary of each 32-edge chunk by
// warp votes.  After a barrier of the 224 workers, work unit u = w, w + 224, ...
// writes the Gaussians 8 (u / TE) .. 8 (u / TE) + 7 of edge u % TE as hi/lo 16-bit
// K-major B rows; in the backward tile row TE + e holds the d-derivative of edge
// e's Gaussians, scaled by 1 / (2 ln 2) (the epilogue folds the factor back in).
// Gaussian columns K .. KP-1 meet zero weight rows: the K-groups of 8 wholly past K
// are zeroed once at kernel start and never written here, and the last partial
// group's extra columns take finite Gaussian values.  Masked or padding edges have
// f_c = f_c' = 0, so their Gaussians need no mask (they stay finite).
constexpr int NWK = GT - 32;              // stage-R workers per group

// named barrier of the stage-R workers of group g (ids 5 and 6)
__device__ __forceinline__ void workers_sync(int g)
{
    asm volatile("bar.sync %0, %1;" ::"r"(5 + g), "n"(NWK) : "memory");
}

template <int FMT, int NX, bool BWD, int TE>
__device__ __forceinline__ void stage_rbf(const MPArgs& a, uint8_t* rbf, TileMeta<TE, BWD>* tmeta, const EdgePre& ep,
                                          int ne, int w, int g)
{
    if (w < TE) {
        const int e = w;
        float d = 0.f, fc = 0.f, dfc = 0.f;
        if (e < ne) {
            d = ep.d;
            if (d < a.rc && d > 0.f) {   // holds for every compacted edge
                float sn, cs;
                sincospif(d * a.inv_rc, &sn, &cs);
                fc = 0.5f * (cs + 1.0f);
                dfc = -0.5f * 3.14159265358979f * a.inv_rc * sn;
            }
        }
        const int row = e < ne ? ep.i : 0x7fffffff;
        tmeta->col[e] = e < ne ? ep.j : 0;
        tmeta->fc[e] = fc;
        tmeta->d[e] = d;
        if (BWD) tmeta->dfc[e] = dfc;
        // the worker's warp holds edges 32c .. 32c+31: summarise the chunk's rows
        const int lane = w & 31, c = e >> 5;
        const int nv = min(max(ne - 32 * c, 0), 32);
        const int rfirst = __shfl_sync(0xffffffffu, row, 0);
        const int rlast = __shfl_sync(0xffffffffu, row, nv > 0 ? nv - 1 : 0);
        const unsigned fm = __ballot_sync(0xffffffffu, e < ne && row == rfirst);
        const int oth = __any_sync(0xffffffffu, e < ne && row != rfirst && row != rlast);
        if (lane == 0) tmeta->c[c] = ChunkInfo{rfirst, rlast, fm, oth};
    }
    workers_sync(g);
    uint8_t* b_hi = rbf;
    uint8_t* b_lo = rbf + RBF_TERM;
    const int nu = TE * ((a.K + 7) >> 3);  // units that hold a Gaussian below K
#pragma unroll 1
    for (int u = w; u < nu; u += NWK) {
        const int e = u & (TE - 1), kg = u / TE;
        const uint32_t off = kmajor_off(e, kg * 8, MN);
        const uint32_t offd = kmajor_off(TE + e, kg * 8, MN);
        const float dm = tmeta->d[e] - fmaf((float)(kg * 8), a.dmu, a.mu0);   // d - mu of the unit's first Gaussian
        float gv[8], dv[8];
        if (!BWD) {
#pragma unroll
            for (int q = 0; q < 8; q += 2) {
                const float2 x = fma2(make_float2(-(float)q, -(float)(q + 1)), dup2(a.dmu), dup2(dm));
                const float2 t = mul2(x, dup2(a.ngc));
                const float2 ee = mul2(t, x);
                gv[q] = ex2_mufu(ee.x);
                gv[q + 1] = ex2_mufu(ee.y);
            }
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float x = fmaf(-(float)q, a.dmu, dm);
                const float t = x * a.ngc;
                const float gg = ex2_mufu(t * x);
                gv[q] = gg;
                dv[q] = t * gg;
            }
        }
        store8_act<FMT, NX>(b_hi, b_lo, off, gv);
        if (BWD) store8_act<FMT, NX>(b_hi, b_lo, offd, dv);
    }
}

// Issue D = W^T * B over KSTEPS K-steps of 16 with the hi/lo split (A: the
// weight term in TMEM, 8 columns per K-step; B: MN = 128 rows in shared
// memory, no-swizzle core matrices).  The small correction products (lo
// weight x hi operand, hi weight x lo operand) are issued first and the
// hi x hi products last: the tensor core's fp32 accumulation does not round
// to nearest, so each MMA added to an accumulator that already holds the large
// sum costs accuracy, and this order keeps those additions to one per K-step.
// The two B descriptors are built once; a K-step advances only their 14-bit
// start-address field (operand regions lie below 256 KB, so the field cannot
// carry into the strides).
template <int NW, int NX, int KSTEPS>
__device__ __forceinline__ void issue_gemm(uint32_t d_tmem, uint32_t a_hi_t, uint32_t a_lo_t, uint32_t b_base,
                                           uint32_t b_term, uint32_t idesc)
{
    const uint64_t bh0 = smem_desc(b_base, MN * 16, 128);
    const uint64_t bl0 = smem_desc(b_base + b_term, MN * 16, 128);
    constexpr bool corr = NW == 2 || NX == 2;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
        const uint64_t step = (uint64_t)((ks * 2 * MN * 16) >> 4);   // 2 core matrices of 8 along K
        if (NW == 2) mma_f16_ts(d_tmem, a_lo_t + ks * 8, bh0 + step, idesc, ks > 0 ? 1u : 0u);
        // the activation residual term is stored negated: its MMA negates B
        if (NX == 2) mma_f16_ts(d_tmem, a_hi_t + ks * 8, bl0 + step, idesc | IDESC_NEG_B, (NW == 2 || ks > 0) ? 1u : 0u);
    }
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
        const uint64_t step = (uint64_t)((ks * 2 * MN * 16) >> 4);
        mma_f16_ts(d_tmem, a_hi_t + ks * 8, bh0 + step, idesc, (corr || ks > 0) ? 1u : 0u);
    }
}

// Wait for group g's tensor-core commit; returns false (uniformly over the
// group) on timeout, leaving `phase` at the commit still outstanding.  The
// group's first warp polls, the others wait at the group barrier.
__device__ __forceinline__ bool wait_mma(uint64_t* bar, uint32_t& phase, DevMeta* meta, int g, int mt)
{
    bool ok = true;
    if ((mt >> 5) == 0) ok = mbar_wait_bounded(bar, phase, WAIT_POLLS);
    if (group_or(g, !ok)) {
        if (mt == 0) set_flag(meta, SCHNET_FLAG_TIMEOUT);
        return false;
    }
    phase ^= 1u;
    tc_fence_after();
    return true;
}

// Wait for group g's tensor-core commit and, for every tile but the first, for the
// epilogue-1 token of the previous tile (phase `tparity`: the other group has
// finished its epilogue 1, which keeps the two groups' MUFU-bound epilogues 1 from
// overlapping and the groups from falling into step); false (uniformly over the
// group) on timeout.  The token orders work only, it guards no data.
__device__ __forceinline__ bool wait_mma_e1(uint64_t* bar, uint32_t& phase, uint64_t* tok, uint32_t tparity,
                                            bool need_tok, DevMeta* meta, int g, int mt)
{
    bool ok = true;
    if ((mt >> 5) == 0) {
        ok = mbar_wait_bounded(bar, phase, WAIT_POLLS);
        if (ok && need_tok) ok = mbar_wait_bounded(tok, tparity, WAIT_POLLS);
    }
    if (group_or(g, !ok)) {
        if (mt == 0) set_flag(meta, SCHNET_FLAG_TIMEOUT);
        return false;
    }
    phase ^= 1u;
    tc_fence_after();
    return true;
}

// Group-uniform bounded wait for phase `parity` of mbarrier `bar` (no wait when
// !need).  Threads with `acquire` repeat the test after the decision, which
// gives each of them its own acquire of what was released before the arrival.
__device__ __forceinline__ bool wait_group(uint64_t* bar, uint32_t parity, bool need, bool acquire, DevMeta* meta,
                                           int g, int mt)
{
    bool ok = true;
    if (need && (mt >> 5) == 0) ok = mbar_wait_bounded(bar, parity, WAIT_POLLS);
    if (group_or(g, !ok)) {
        if (mt == 0) set_flag(meta, SCHNET_FLAG_TIMEOUT);
        return false;
    }
    if (need && acquire && (mt >> 5) != 0) (void)mbar_try_wait(bar, parity);
    return true;
}

// x_j,f (one feature per thread, src_f = x + f) for N consecutive edges starting at e;
// the column indices come four at a time from the tile's column array
template <int N>
__device__ __forceinline__ void gather(const float* __restrict__ src_f, const int32_t* col, int e, float (&dst)[N])
{
#pragma unroll
    for (int q = 0; q < N; q += 4) {
        const int4 j = *reinterpret_cast<const int4*>(col + e + q);
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

// A completed row's sum into out, and zeros for the rows without edges between two
// rows with edges (every row of the CTA's range is written).
__device__ __forceinline__ void put_row(float* __restrict__ out, int row, int f, float v)
{
    out[(size_t)row * FP + f] = v;
}
__device__ __forceinline__ void zero_rows(float* __restrict__ out, int from, int to, int f)
{
    for (int rr = from; rr < to; ++rr) out[(size_t)rr * FP + f] = 0.f;
}

__device__ __forceinline__ void seg_begin(ChunkSeg& c, int rfirst)
{
    c.rfirst = rfirst;
    c.lrow = rfirst;
    c.acc = 0.f;
    c.pf = 0.f;
}

__device__ __forceinline__ void seg_row(ChunkSeg& c, int row, float* __restrict__ out, int f)
{
    if (row != c.lrow) {
        if (c.lrow == c.rfirst) c.pf = c.acc;
        else put_row(out, c.lrow, f, c.acc);
        zero_rows(out, c.lrow + 1, row, f);
        c.lrow = row;
        c.acc = 0.f;
    }
}

// In-order merge of a tile's chunk partials into the carried row (threads of
// the group with feature f = group thread index < 128): rows the carry leaves
// are complete and written out, with zeros for edge-less rows in between.
template <int NCH>
__device__ __forceinline__ void merge_chunks(const ChunkInfo* ci, const float* pf, const float* pl, int ne, int f,
                                             float* __restrict__ out, int& cur, float& acc)
{
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        if (c * 32 >= ne) break;
        const int rfirst = ci[c].rfirst, rlast = ci[c].rlast;
        const float v = pf[c * 128 + f];
        if (rfirst == cur) {
            acc += v;
        } else {
            put_row(out, cur, f, acc);
            zero_rows(out, cur + 1, rfirst, f);
            cur = rfirst;
            acc = v;
        }
        if (rlast != rfirst) {
            put_row(out, cur, f, acc);
            cur = rlast;
            acc = pl[c * 128 + f];
        }
    }
}

// Merge step of tile t by its group's warps 0-3 (thread mt = feature): wait for
// tile t-1's merge (warp 0 polls the token, a barrier of the 128 merging threads
// shares the outcome, and warps 1-3 repeat the test for their own acquire), fold
// this tile's partials into the carry, hand the carry on.  Returns false (uniformly
// over the 128 threads) on timeout.
template <int NCH>
__device__ __forceinline__ bool merge_tile(Carry* cy, uint64_t* tok, const ChunkInfo* ci, const float* pf,
                                           const float* pl, int ne, int t, float* __restrict__ out, DevMeta* meta,
                                           int g, int mt)
{
    if (t > 0) {
        const uint32_t parity = (uint32_t)((t - 1) & 1);
        bool ok = true;
        if ((mt >> 5) == 0) ok = mbar_wait_bounded(tok, parity, WAIT_POLLS);
        if (merge_or(g, !ok)) {
            if (mt == 0) set_flag(meta, SCHNET_FLAG_TIMEOUT);
            return false;
        }
        if ((mt >> 5) != 0) (void)mbar_try_wait(tok, parity);
    }
    int cur = cy->cur[(t + 1) & 1];      // written by tile t-1 (or the initial row)
    float acc = cy->acc[mt];
    merge_chunks<NCH>(ci, pf, pl, ne, mt, out, cur, acc);
    cy->acc[mt] = acc;
    if (mt == 0) cy->cur[t & 1] = cur;
    mbar_arrive(tok);
    return true;
}

// pairwise sum of N values (fixed order)
template <int N>
__device__ __forceinline__ float tree_sum(float (&v)[N])
{
#pragma unroll
    for (int w = N / 2; w >= 2; w >>= 1)
#pragma unroll
        for (int q = 0; q < w; q += 2) {
            const float2 t = add2(make_float2(v[q], v[q + 1]), make_float2(v[q + w], v[q + w + 1]));
            v[q] = t.x;
            v[q + 1] = t.y;
        }
    return v[0] + v[1];
}

// Reduce a chunk's per-edge terms t[q] (edge eb + q) to the first-row and
// last-row partials.  One or two rows: branch-free predicated sums (edge-less
// rows strictly between them are written as zeros).  Three or more rows: the
// serial segmented sum (rows read from the tile's global row list) writes the
// inner rows out.
template <int N>
__device__ __forceinline__ void chunk_partials(const ChunkInfo& ci, const int32_t* __restrict__ rows_g, int eb,
                                               int ne, float (&t)[N], float* __restrict__ out, int f, float& pf,
                                               float& pl)
{
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
            zero_rows(out, ci.rfirst + 1, ci.rlast, f);
        }
        return;
    }
    ChunkSeg c;
    seg_begin(c, ci.rfirst);
#pragma unroll
    for (int q = 0; q < N; ++q) {
        const int e = eb + q;
        if (e >= ne) break;
        seg_row(c, __ldg(rows_g + e), out, f);
        c.acc += t[q];
    }
    if (c.lrow == c.rfirst) { pf = c.acc; pl = 0.f; } else { pf = c.pf; pl = c.acc; }
}

// Common prologue of both kernels, on constant data only (it runs before
// pdl_wait): TMEM allocation, mbarriers, the filter weights into TMEM (one output
// channel per lane; the six 32-column row loads of each lane quadrant spread over
// the quadrant's four warps), the zero carry.  Returns the TMEM base address.
__device__ __forceinline__ uint32_t kernel_setup(const MPArgs& a, uint8_t* smem, uint32_t* tslot, uint64_t* bars,
                                                 Carry* cy)
{
    const int warp = threadIdx.x >> 5;
    {
        // the K-groups of both groups' GEMM1 B operands (hi and lo terms) wholly past K: zero
        // for every tile, so stage R does not write them
        const int nkg = (a.K + 7) >> 3;
        const uint32_t pad = (uint32_t)(KP / 8 - nkg) * (MN * 16);   // bytes per term
        for (uint32_t o = threadIdx.x * 16; o < 4 * pad; o += NT * 16) {
            const uint32_t term = o / pad, r = o % pad;                // term = 2 group + (hi, lo)
            *reinterpret_cast<uint4*>(smem + SM_RBF + term * RBF_TERM + (uint32_t)nkg * (MN * 16) + r) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);      // group 0 MMA commits
        mbar_init(&bars[1], 1);      // group 1 MMA commits
        mbar_init(&bars[2], 128);    // merge token: the 128 merging threads of a tile
        mbar_init(&bars[3], 1);      // group 1 start
        mbar_init(&bars[4], 1);      // epilogue-1 token: one arrival per tile, in tile order
        fence_mbar_init();
    }
    if (threadIdx.x < FP) cy->acc[threadIdx.x] = 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    {
        const int qd = warp & 3;                      // the lane quadrant this warp may access
        const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
        const int f = qd * 32 + (threadIdx.x & 31);
        // job j: 0 W1 hi, 1 W1 lo, 2-3 W2 hi (K halves), 4-5 W2 lo; warp takes jobs warp/4 and
        // warp/4 + 4, both rows loaded before either store (one trip to L2)
        auto col_of = [](int j) { return j == 0 ? TM_W1H : j == 1 ? TM_W1L : j < 4 ? TM_W2H : TM_W2L; };
        auto term_of = [&](int j) {
            return a.img + (j == 0 ? 0 : j == 1 ? W1_IMG : j < 4 ? 2 * W1_IMG : 2 * W1_IMG + W2_IMG);
        };
        auto half_of = [](int j) { return j < 2 ? 0 : j & 1; };
        const int j0 = warp >> 2, j1 = j0 + NT / 128;
        uint32_t v0[32], v1[32];
        weight_row(term_of(j0), f, half_of(j0), v0);
        if (j1 < 6) weight_row(term_of(j1), f, half_of(j1), v1);
        tmem_st32(tl + col_of(j0) + half_of(j0) * 32, v0);
        if (j1 < 6) tmem_st32(tl + col_of(j1) + half_of(j1) * 32, v1);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return tmem;
}

// This CTA's row range [r0, r1), empty when the list overflowed its capacity.
// Read before pdl_wait: the partitions and the edge count are written only by the
// neighbour build, whose kernels are launched without programmatic serialization,
// so they have completed before any kernel of a step or evaluation starts.  A CTA
// without rows returns at once, before it allocates tensor memory.
__device__ __forceinline__ void kernel_rows(const MPArgs& a, int& r0, int& r1)
{
    r0 = r1 = 0;
    if (a.meta->n_edges <= a.cap) {
        r0 = a.part[blockIdx.x];
        r1 = a.part[blockIdx.x + 1];
    }
}

// Common epilogue: the carried row is complete; rows after it without edges are zero
// (nothing to write when the kernel produces no per-row output).
__device__ __forceinline__ void kernel_finish(const Carry* cy, int ntiles, int r1, float* __restrict__ out, bool ok,
                                              uint64_t* bars, const uint32_t* phases, const uint32_t* pending,
                                              uint32_t tmem, bool write_out = true)
{
    const int warp = threadIdx.x >> 5;
    if (ok && write_out) {
        if (threadIdx.x < FP) {
            const int cur = cy->cur[(ntiles + 1) & 1];
            if (ntiles > 0) put_row(out, cur, threadIdx.x, cy->acc[threadIdx.x]);
            else zero_rows(out, cur, cur + 1, threadIdx.x);
            zero_rows(out, cur + 1, r1, threadIdx.x);
        }
    } else if ((threadIdx.x & (GT - 1)) == 0) {
        // drain: give the group's in-flight MMAs a bounded chance to retire before freeing TMEM
        const int g = threadIdx.x / GT;
        if (pending[g]) mbar_wait_bounded(&bars[g], phases[g], WAIT_POLLS);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// forward epilogue 1 for 32 edges: a = ssp2(s1 log2e P + b1 log2e) -> MN-major B
// operand (the base-2 shifted softplus: ssp = ln2 a, with ln2 folded into the
// second layer's scale).  With one 16-bit activation term (NX = 1) the operand is
// sp2 = ssp2 + 1 instead, and the -1 is folded into the second layer's bias.
template <int FMT, int NX>
__device__ __forceinline__ void fwd_e1(uint32_t tP, float s1L, float b1L, uint8_t* act, int e0, int f)
{
    float r[32];
    tmem_ld32(tP, r);
    tmem_ld_wait();
#pragma unroll
    for (int q = 0; q < 32; q += 2) {
        // one pair in four takes its exponentials on the FMA pipe: the MUFU, which the
        // logarithms and the other exponentials keep busy, is this epilogue's bottleneck
        const float2 pp = fma2(dup2(s1L), make_float2(r[q], r[q + 1]), dup2(b1L));
        const float2 v = ((q >> 1) & 3) == 3 ? sp2x2_fma<NX == 2>(pp) : sp2x2<NX == 2>(pp);
        r[q] = v.x;
        r[q + 1] = v.y;
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const uint32_t off = mnmajor_off(e0 + g * 8, f, MN);
        store8_act<FMT, NX>(act, act + ACT_TERM, off, r + g * 8);
    }
}

// forward epilogue 2 for chunk cc: W = f_c (s2 ln2 Q + b2), terms h_j W, chunk partials
template <int TE>
__device__ __forceinline__ void fwd_e2(uint32_t tQ, const TileMeta<TE, false>* tm, const int32_t* rows_g, int cc,
                                       int ne, float s2L, float b2, const float (&hv)[32], float* __restrict__ out,
                                       int f, float& pf, float& pl)
{
    float r[32];
    tmem_ld32(tQ, r);
    tmem_ld_wait();
    const int eb = cc * 32;
    pf = pl = 0.f;
    if (eb >= ne) return;
    float fc[32];
    load_edges<32>(tm->fc, eb, fc);
#pragma unroll
    for (int q = 0; q < 32; q += 2) {
        const float2 z = fma2(dup2(s2L), make_float2(r[q], r[q + 1]), dup2(b2));
        const float2 v = mul2(mul2(make_float2(fc[q], fc[q + 1]), z), make_float2(hv[q], hv[q + 1]));
        r[q] = v.x;
        r[q + 1] = v.y;
    }
    chunk_partials<32>(tm->c[cc], rows_g, eb, ne, r, out, f, pf, pl);
}

// Issue GEMM1 of a tile (group g): D = W1^T [B rows of the group's GEMM1 operand]
template <int NW, int NX>
__device__ __forceinline__ void issue_gemm1(uint32_t tmem, uint32_t dacc, uint32_t srbf, uint32_t id, uint64_t* bar)
{
    tc_fence_after();
    issue_gemm<NW, NX, KP / 16>(dacc, tmem + TM_W1H, tmem + TM_W1L, srbf, RBF_TERM, id);
    mma_commit(bar);
}

// ---------------------------------------------------------------------------
// forward: m_i = sum_j h_j (.) W(d_ij)
// ---------------------------------------------------------------------------
// Per group and tile t: [GEMM1(t) in flight] E1 -> issue GEMM2 (warp 0) -> stage R
// of t+2 (warps 1-7, into the group's own GEMM1 operand and second metadata
// buffer) and the first gather under GEMM2 -> E2 -> issue GEMM1(t+2) (warp 4) ->
// merge under GEMM1(t+2) (warps 0-3).
template <int FMT, int NW, int NX>
__global__ void __launch_bounds__(NT, 1) k_cfconv_fwd(MPArgs a)
{
    constexpr int TE = TE_F;
    constexpr int NCH = TE / 32;
    using Meta = TileMeta<TE, false>;
    extern __shared__ __align__(1024) uint8_t smem[];
    Carry* cy = reinterpret_cast<Carry*>(smem + sm_carry<TE, false>());
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sm_bar<TE, false>());
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 5);
    uint32_t* phases_s = tslot + 1;
    uint32_t* pend_s = tslot + 3;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = warp >> 3;                        // math group
    const int mt = threadIdx.x & (GT - 1);          // thread within the group
    const int qd = warp & 3, ch = (warp >> 2) & 1;  // TMEM lane quadrant, 64-edge half of the tile
    const int f = qd * 32 + lane;                   // this thread's output feature

    pdl_trigger();
    int r0, r1;
    kernel_rows(a, r0, r1);
    if (r0 >= r1) return;
    const uint32_t tmem = kernel_setup(a, smem, tslot, bars, cy);
    if (threadIdx.x == 0) cy->cur[1] = r0;         // tile 0 reads the carry of "tile -1"
    pdl_wait();                                     // the previous kernel's results from here on
    __syncthreads();
    const long long e0 = a.row_ptr[r0], e1 = e0 + a.ccount[blockIdx.x];
    uint8_t* rbf = smem + SM_RBF + g * 2 * RBF_TERM;
    uint8_t* act = smem + SM_ACT + g * 2 * ACT_TERM;
    Meta* tmb = reinterpret_cast<Meta*>(smem + sm_meta<TE, false>() + g * 2 * sizeof(Meta));
    float* pf_s = reinterpret_cast<float*>(act);    // after GEMM2: [chunk][feature] partials
    float* pl_s = pf_s + NCH * 128;
    const uint32_t dacc = tmem + g * TM_ACC;        // P, then Q over it (128 columns)
    const uint32_t tA = dacc + ((uint32_t)(qd * 32) << 16) + ch * 64;
    const uint32_t srbf = smem_u32(rbf), sact = smem_u32(act);
    const uint32_t id = idesc_f16(128, MN, FMT, 0);
    const uint32_t id_mn = idesc_f16(128, MN, FMT, 1);
    const float s1L = a.s1[f] * LOG2EF, b1L = a.b1[f] * LOG2EF;
    const float s2L = a.s2[f] * LN2F, b2 = a.b2[f];
    const float* h_f = a.h + f;

    uint32_t phase = 0, pending = 0;   // pending: a commit of this group not yet waited for
    bool ok = true, go_sent = false;
    const int ntiles = (int)((e1 - e0 + TE - 1) / TE);
    auto tile_ne = [&](int t) { return (int)min((long long)TE, e1 - e0 - (long long)t * TE); };

    const int w = mt - 32;                          // stage-R worker (warps 1-7 of the group)
    EdgePre ep;
    if (g < ntiles) {
        if (g == 1) ok = wait_group(&bars[3], 0u, true, false, a.meta, g, mt);   // start half a tile behind
        ep = prefetch_edge<TE, false>(a, e0 + (long long)g * TE, tile_ne(g), w);
        if (w >= 0) stage_rbf<FMT, NX, false, TE>(a, rbf, tmb, ep, tile_ne(g), w, g);
        if (g + 2 < ntiles) ep = prefetch_edge<TE, false>(a, e0 + (long long)(g + 2) * TE, tile_ne(g + 2), w);
        fence_proxy_async_smem();
        tc_fence_before();
        group_sync(g);
        if (ok && mt == 0) issue_gemm1<NW, NX>(tmem, dacc, srbf, id, &bars[g]);
        pending = ok ? 1 : 0;
    }
    int buf = 0;
    for (int t = g; t < ntiles && ok; t += 2, buf ^= 1) {
        const int ne = tile_ne(t);
        const bool next = t + 2 < ntiles;
        Meta* tm = tmb + buf;
        const int32_t* rows_g = a.crow + e0 + (long long)t * TE;
        // GEMM1(t) done (the epilogue-1 token is not used here: with it the forward settles
        // a quarter tile apart, as without, and runs 0.5 % slower)
        if (!(ok = wait_mma_e1(&bars[g], phase, &bars[4], 0u, false, a.meta, g, mt))) break;
        pending = 0;
        if (g == 0 && !go_sent) {
            if (mt == 0) mbar_arrive(&bars[3]);
            go_sent = true;
        }
#pragma unroll 1
        for (int c2 = 0; c2 < 2; ++c2) fwd_e1<FMT, NX>(tA + c2 * 32, s1L, b1L, act, ch * 64 + c2 * 32, f);
        fence_proxy_async_smem();
        tc_fence_before();
        group_sync(g);
        if (mt == 0) {
            tc_fence_after();
            issue_gemm<NW, NX, FP / 16>(dacc, tmem + TM_W2H, tmem + TM_W2L, sact, ACT_TERM, id_mn);
            mma_commit(&bars[g]);
        }
        pending = 1;
        // under GEMM2: stage R of tile t+2 (warps 1-7) and the first gather of this tile
        if (next) {
            if (w >= 0) stage_rbf<FMT, NX, false, TE>(a, rbf, tmb + (buf ^ 1), ep, tile_ne(t + 2), w, g);
            if (t + 4 < ntiles) ep = prefetch_edge<TE, false>(a, e0 + (long long)(t + 4) * TE, tile_ne(t + 4), w);
            fence_proxy_async_smem();
        }
        float hv[32];
        gather<32>(h_f, tm->col, ch * 64, hv);
        if (!(ok = wait_mma(&bars[g], phase, a.meta, g, mt))) break;     // GEMM2(t) done
        pending = 0;
#pragma unroll 1
        for (int c2 = 0; c2 < 2; ++c2) {
            const int cc = ch * 2 + c2;
            if (c2 == 1) gather<32>(h_f, tm->col, cc * 32, hv);
            float pf, pl;
            fwd_e2<TE>(tA + c2 * 32, tm, rows_g, cc, ne, s2L, b2, hv, a.out, f, pf, pl);
            pf_s[cc * 128 + f] = pf;
            pl_s[cc * 128 + f] = pl;
        }
        tc_fence_before();
        group_sync(g);          // Q read out; partials and the next tile's Gaussians in place
        // GEMM1(t+2) is issued by warp 4, which takes no part in the merge below (an issuing
        // thread blocks while the tensor core's queue is full)
        if (next && mt == 128) issue_gemm1<NW, NX>(tmem, dacc, srbf, id, &bars[g]);
        if (next) pending = 1;
        bool merged = true;
        if (mt < 128) merged = merge_tile<NCH>(cy, &bars[2], tm->c, pf_s, pl_s, ne, t, a.out, a.meta, g, mt);
        // the merge done with the partials before E1 of the next tile overwrites them (and its
        // outcome known to the whole group)
        if (!(ok = !group_or(g, !merged))) break;
    }
    if (g == 0 && !go_sent && mt == 0) mbar_arrive(&bars[3]);
    if (mt == 0) {
        phases_s[g] = phase;
        pend_s[g] = ok ? 0u : pending;
    }
    const bool all_ok = __syncthreads_or(!ok) == 0;
    kernel_finish(cy, ntiles, r1, a.out, all_ok, bars, phases_s, pend_s, tmem);
}

// ---------------------------------------------------------------------------
// backward: dh_i = sum_j u_j (.) W_ij ;  s_e = sum_f W'_e,f u_i,f h_j,f
// ---------------------------------------------------------------------------
// backward epilogue 1 for this warp's 32 edges: a = ssp2(p), b = ssp'(x) dx/dd, with
// p = x log2e = s1 log2e P + b1 log2e and dx/dd = s1 2ln2 P' (P' from the scaled
// Gaussian-derivative rows).  With t = 2^-|p| and l = log2((1 + t) / 2) (the
// logarithm ssp2 takes anyway), the logistic ssp'(x) = 1 / (1 + e^-x) is
// 2^-l / 2 for p >= 0 and t 2^-l / 2 for p < 0: one more exponential, no
// division and no cancellation; the factor 1/2 is folded into s1d.  With one
// 16-bit activation term (NX = 1) a is sp2 = ssp2 + 1 and l = log2(1 + t) (see
// the forward epilogue), and s1d has no factor 1/2.
// a goes to B rows e, b to B rows TE + e of GEMM2's operand.  Pairs of
// elements share the packed fp32x2 FMA/FMUL/FADD instructions.
template <int FMT, int NX, int TE>
__device__ __forceinline__ void bwd_e1(uint32_t tP, uint32_t tPd, float s1L, float b1L, float s1d, uint8_t* act,
                                       int col0, int f)
{
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float r[16], rd[16];
        tmem_ld16(tP + hh * 16, r);
        tmem_ld16(tPd + hh * 16, rd);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 16; q += 2) {
            const float2 p = fma2(dup2(s1L), make_float2(r[q], r[q + 1]), dup2(b1L));
            // one pair in four takes 2^-|p| from the FMA pipe (the MUFU carries three operations
            // per element here)
            const float2 t = ((q >> 1) & 3) == 3 ? ex2_fma2(make_float2(-fabsf(p.x), -fabsf(p.y)))
                                                 : make_float2(ex2_mufu(-fabsf(p.x)), ex2_mufu(-fabsf(p.y)));
            constexpr float c = NX == 2 ? 0.5f : 1.0f;
            const float2 y = fma2(dup2(c), t, dup2(c));                     // c (1 + t)
            const float2 l = make_float2(lg2_mufu(y.x), lg2_mufu(y.y));
            const float2 g = make_float2(ex2_mufu(-l.x), ex2_mufu(-l.y));   // 1 / (c (1 + t))
            const float2 sg = mul2(make_float2(p.x >= 0.0f ? 1.0f : t.x, p.y >= 0.0f ? 1.0f : t.y), g);
            const float2 a = add2(make_float2(fmaxf(p.x, 0.0f), fmaxf(p.y, 0.0f)), l);
            const float2 d = mul2(sg, mul2(dup2(s1d), make_float2(rd[q], rd[q + 1])));
            r[q] = a.x;
            r[q + 1] = a.y;
            rd[q] = d.x;
            rd[q + 1] = d.y;
        }
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            const int e = col0 + hh * 16 + g * 8;
            store8_act<FMT, NX>(act, act + ACT_TERM, mnmajor_off(e, f, MN), r + g * 8);
            store8_act<FMT, NX>(act, act + ACT_TERM, mnmajor_off(TE + e, f, MN), rd + g * 8);
        }
    }
}

// Backward of one interaction.  The pair derivative
// dE/dd_ij = D_ij = sum_f W'_f(d_ij) (u_i,f h_j,f + u_j,f h_i,f) is the same for
// (i, j) and (j, i) because W_ij = W_ji: the launch runs over one edge per
// unordered pair (the half list: the edges (i, j) that own their pair, in rows
// balanced by their own partition) and writes (adds, for the later interactions'
// sums) D_ij to s_e of that edge; the force assembly reads each pair's value from
// its owning edge, so both atoms receive it.  With DH (every interaction but the
// first, whose dE/dh would only reach the embedding) the same tiles also form
// row i's share of dE/dh_i = sum_j W_ij (.) u_j over its half-list edges, a
// segment sum in registers written to out like the forward's; the other terms
// (the complement's edges) come from the forward kernel over the complementary
// list, in a second buffer.
template <int FMT, int NW, int NX, bool DH>
__global__ void __launch_bounds__(NT, 1) k_cfconv_bwd(MPArgs a)
{
    constexpr int TE = TE_B;
    constexpr int NCH = TE / 32;
    using Meta = TileMeta<TE, true>;
    extern __shared__ __align__(1024) uint8_t smem[];
    Carry* cy = reinterpret_cast<Carry*>(smem + sm_carry<TE, true>());
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sm_bar<TE, true>());
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 5);
    uint32_t* phases_s = tslot + 1;
    uint32_t* pend_s = tslot + 3;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = warp >> 3;
    const int mt = threadIdx.x & (GT - 1);
    const int qd = warp & 3, ch = (warp >> 2) & 1;  // TMEM lane quadrant, 32-edge chunk of the tile
    const int f = qd * 32 + lane;

    pdl_trigger();
    int r0, r1;
    kernel_rows(a, r0, r1);
    if (r0 >= r1) return;
    const uint32_t tmem = kernel_setup(a, smem, tslot, bars, cy);
    if (threadIdx.x == 0) cy->cur[1] = r0;         // tile 0 reads the carry of "tile -1"
    pdl_wait();                                     // the previous kernel's results from here on
    __syncthreads();
    const long long e0 = a.row_ptr[r0], e1 = e0 + a.ccount[blockIdx.x];
    uint8_t* rbf = smem + SM_RBF + g * 2 * RBF_TERM;
    uint8_t* act = smem + SM_ACT + g * 2 * ACT_TERM;
    Meta* tmb = reinterpret_cast<Meta*>(smem + sm_meta<TE, true>() + g * 2 * sizeof(Meta));
    float* pf_s = reinterpret_cast<float*>(act);    // after GEMM2: [chunk][feature] dE/dh partials
    float* pl_s = pf_s + NCH * 128;
    float* ps_s = pl_s + NCH * 128;                 // [quadrant][edge] partial of D
    // per-warp [32 edges][36] scratch of the D transpose (behind the partials, inside the
    // group's GEMM2 operand buffer, which is free between GEMM2's completion and the next E1)
    float* s_w = reinterpret_cast<float*>(act + 4096) + (warp & 7) * (32 * 36);
    const int col0 = ch * 32;
    // accumulator columns: [P | P'] (64 each), then [Q | Q'] over them
    const uint32_t dacc = tmem + g * TM_ACC;
    const uint32_t tP = dacc + ((uint32_t)(qd * 32) << 16) + col0, tPd = tP + 64;
    const uint32_t srbf = smem_u32(rbf), sact = smem_u32(act);
    const uint32_t id = idesc_f16(128, MN, FMT, 0);
    const uint32_t id_mn = idesc_f16(128, MN, FMT, 1);
    const float s1L = a.s1[f] * LOG2EF, b1L = a.b1[f] * LOG2EF, s1d = a.s1[f] * (NX == 2 ? LN2F : 2.0f * LN2F);
    const float s2 = a.s2[f], s2L = a.s2[f] * LN2F, b2 = a.b2[f];
    const float* h_f = a.h + f;
    const float* u_f = a.u + f;

    uint32_t phase = 0, pending = 0;   // pending: a commit of this group not yet waited for
    bool ok = true, go_sent = false;
    const int ntiles = (int)((e1 - e0 + TE - 1) / TE);
    auto tile_ne = [&](int t) { return (int)min((long long)TE, e1 - e0 - (long long)t * TE); };

    const int w = mt - 32;         // stage-R worker (warps 1-7 of the group)
    EdgePre ep;
    int my_g = 0, nx_g = 0;        // workers w < TE: s_e slot of edge w (this tile / tile t+2)
    float my_so = 0.f, nx_so = 0.f;
    if (g < ntiles) {
        if (g == 1) ok = wait_group(&bars[3], 0u, true, false, a.meta, g, mt);   // start half a tile behind
        ep = prefetch_edge<TE, true>(a, e0 + (long long)g * TE, tile_ne(g), w);
        if (w >= 0) stage_rbf<FMT, NX, true, TE>(a, rbf, tmb, ep, tile_ne(g), w, g);
        nx_g = ep.gidx;
        nx_so = ep.sold;
        if (g + 2 < ntiles) ep = prefetch_edge<TE, true>(a, e0 + (long long)(g + 2) * TE, tile_ne(g + 2), w);
        fence_proxy_async_smem();
        tc_fence_before();
        group_sync(g);
        if (ok && mt == 0) issue_gemm1<NW, NX>(tmem, dacc, srbf, id, &bars[g]);
        pending = ok ? 1 : 0;
    }
    int buf = 0;
    for (int t = g; t < ntiles && ok; t += 2, buf ^= 1) {
        const int ne = tile_ne(t);
        const bool next = t + 2 < ntiles;
        Meta* tm = tmb + buf;
        const int32_t* rows_g = a.crow + e0 + (long long)t * TE;
        my_g = nx_g;
        my_so = nx_so;
        // GEMM1(t) done, and epilogue 1 of tile t-1 (the other group's)
        if (!(ok = wait_mma_e1(&bars[g], phase, &bars[4], (uint32_t)((t - 1) & 1), t > 0, a.meta, g, mt))) break;
        pending = 0;
        if (g == 0 && !go_sent) {
            if (mt == 0) mbar_arrive(&bars[3]);
            go_sent = true;
        }
        bwd_e1<FMT, NX, TE>(tP, tPd, s1L, b1L, s1d, act, col0, f);
        fence_proxy_async_smem();
        tc_fence_before();
        group_sync(g);
        if (mt == 0) {
            mbar_arrive(&bars[4]);  // epilogue 1 of tile t done: the other group's tile t+1 may start its own
            tc_fence_after();
            issue_gemm<NW, NX, FP / 16>(dacc, tmem + TM_W2H, tmem + TM_W2L, sact, ACT_TERM, id_mn);
            mma_commit(&bars[g]);
        }
        pending = 1;
        // under GEMM2: stage R of tile t+2 (warps 1-7) and the first gathers of this tile
        if (next) {
            if (w >= 0) stage_rbf<FMT, NX, true, TE>(a, rbf, tmb + (buf ^ 1), ep, tile_ne(t + 2), w, g);
            nx_g = ep.gidx;
            nx_so = ep.sold;
            if (t + 4 < ntiles) ep = prefetch_edge<TE, true>(a, e0 + (long long)(t + 4) * TE, tile_ne(t + 4), w);
            fence_proxy_async_smem();
        }
        const int eb = col0;
        float uv[16], hv[16];
        gather<16>(u_f, tm->col, eb, uv);
        gather<16>(h_f, tm->col, eb, hv);
        // u and h of the chunk's first and last rows, shared by all its edges
        float u_first = 0.f, u_last = 0.f, h_first = 0.f, h_last = 0.f;
        if (eb < ne) {
            const int rf = tm->c[ch].rfirst, rl = tm->c[ch].rlast;
            u_first = __ldg(u_f + (size_t)rf * FP);
            u_last = __ldg(u_f + (size_t)rl * FP);
            h_first = __ldg(h_f + (size_t)rf * FP);
            h_last = __ldg(h_f + (size_t)rl * FP);
        }
        if (!(ok = wait_mma(&bars[g], phase, a.meta, g, mt))) break;     // GEMM2(t) done
        pending = 0;
        // epilogue 2: W = f_c z, W' = f_c' z + f_c z' (z = s2 ln2 Q + b2, z' = s2 Q'); per edge the
        // pair derivative D = sum_f W'_f (u_i,f h_j,f + u_j,f h_i,f) and, with DH, the row's share
        // of dE/dh_i = sum_j W_ij (.) u_j as a segment sum (chunk partials, merged in tile order)
        {
            float pf = 0.f, pl = 0.f;
            if (eb < ne) {
                const ChunkInfo ci = tm->c[ch];
                // 1: one row in the chunk; 2: two rows (the first a prefix); 3: a third row
                // occurs, rows read per edge
                const int kind = ci.other ? 3 : (ci.rfirst == ci.rlast ? 1 : 2);
                float u_row = u_first, h_row = h_first;
                float sf = 0.f, sl = 0.f;
                ChunkSeg c;
                seg_begin(c, ci.rfirst);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    if (hh == 1) {
                        gather<16>(u_f, tm->col, eb + 16, uv);
                        gather<16>(h_f, tm->col, eb + 16, hv);
                    }
                    float r[16], rd[16];
                    tmem_ld16(tP + hh * 16, r);          // Q
                    tmem_ld16(tPd + hh * 16, rd);        // Q'
                    tmem_ld_wait();
                    const float* fcp = tm->fc + eb + hh * 16;
                    const float* dfcp = tm->dfc + eb + hh * 16;
                    if (kind == 1) {
#pragma unroll
                        for (int gq = 0; gq < 16; gq += 4) {
                            float fc[4], dfc[4];
                            load_edges<4>(fcp, gq, fc);
                            load_edges<4>(dfcp, gq, dfc);
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int q = gq + i;
                                const float z = fmaf(s2L, r[q], b2);
                                if (DH) sf = fmaf(fc[i] * z, uv[q], sf);
                                const float wd = fmaf(dfc[i], z, fc[i] * (s2 * rd[q]));
                                rd[q] = wd * fmaf(uv[q], h_first, u_first * hv[q]);
                            }
                        }
                    } else if (kind == 2) {
#pragma unroll
                        for (int gq = 0; gq < 16; gq += 4) {
                            float fc[4], dfc[4];
                            load_edges<4>(fcp, gq, fc);
                            load_edges<4>(dfcp, gq, dfc);
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int q = gq + i;
                                const float z = fmaf(s2L, r[q], b2);
                                const bool first = (ci.firstmask >> (hh * 16 + q)) & 1u;
                                if (DH) {
                                    const float dt = fc[i] * z * uv[q];
                                    sf += first ? dt : 0.f;
                                    sl += first ? 0.f : dt;
                                }
                                const float wd = fmaf(dfc[i], z, fc[i] * (s2 * rd[q]));
                                rd[q] = wd * fmaf(uv[q], first ? h_first : h_last, (first ? u_first : u_last) * hv[q]);
                            }
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            const int e = eb + hh * 16 + q;
                            float tval = 0.f;
                            if (e < ne) {
                                const int row = __ldg(rows_g + e);
                                if (row != c.lrow) {
                                    if (DH) seg_row(c, row, a.out, f);
                                    else c.lrow = row;
                                    u_row = __ldg(u_f + (size_t)row * FP);
                                    h_row = __ldg(h_f + (size_t)row * FP);
                                }
                                const float z = fmaf(s2L, r[q], b2);
                                if (DH) c.acc = fmaf(fcp[q] * z, uv[q], c.acc);
                                const float wd = fmaf(dfcp[q], z, fcp[q] * (s2 * rd[q]));
                                tval = wd * fmaf(uv[q], h_row, u_row * hv[q]);
                            }
                            rd[q] = tval;
                        }
                    }
                    // stage this half's 16 per-edge values as S[edge][feature lane] (row stride 36:
                    // the stores and the 16-byte row reads below are free of bank conflicts)
#pragma unroll
                    for (int q = 0; q < 16; ++q) s_w[(hh * 16 + q) * 36 + lane] = rd[q];
                }
                // lane k sums edge k of the warp's chunk over the warp's 32 features (the same
                // pairwise tree as a butterfly over the lanes)
                __syncwarp();
                {
                    float v[32];
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 x = *reinterpret_cast<const float4*>(s_w + lane * 36 + c4 * 4);
                        v[4 * c4] = x.x; v[4 * c4 + 1] = x.y; v[4 * c4 + 2] = x.z; v[4 * c4 + 3] = x.w;
                    }
                    ps_s[qd * TE + eb + lane] = tree_sum<32>(v);
                }
                __syncwarp();
                if (!DH) {
                } else if (kind == 1) {
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
            if (DH) {
                pf_s[ch * 128 + f] = pf;
                pl_s[ch * 128 + f] = pl;
            }
        }
        tc_fence_before();
        group_sync(g);          // Q, Q' read out; per-edge partials and the next tile's Gaussians in place
        // GEMM1(t+2) is issued by warp 4, which does not write s_e below (warps 1 and 2 do; an
        // issuing thread blocks while the tensor core's queue is full)
        if (next && mt == 128) issue_gemm1<NW, NX>(tmem, dacc, srbf, id, &bars[g]);
        if (next) pending = 1;
        if (w >= 0 && w < ne) {
            const float sv = ps_s[w] + ps_s[TE + w] + ps_s[2 * TE + w] + ps_s[3 * TE + w];
            a.s_edge[my_g] = a.accumulate_s ? my_so + sv : sv;
        }
        if (DH) {
            bool merged = true;
            if (mt < 128) merged = merge_tile<NCH>(cy, &bars[2], tm->c, pf_s, pl_s, ne, t, a.out, a.meta, g, mt);
            // s_e and the merge done with the partials before E1 of the next tile overwrites them
            if (!(ok = !group_or(g, !merged))) break;
        } else {
            group_sync(g);      // s_e done with the partials before E1 of the next tile overwrites them
        }
    }
    if (g == 0 && !go_sent && mt == 0) mbar_arrive(&bars[3]);
    if (mt == 0) {
        phases_s[g] = phase;
        pend_s[g] = ok ? 0u : pending;
    }
    const bool all_ok = __syncthreads_or(!ok) == 0;
    kernel_finish(cy, ntiles, r1, a.out, all_ok, bars, phases_s, pend_s, tmem, DH);
}

// ---------------------------------------------------------------------------
// cutoff masking: per CTA row range, the listed edges with d < r_c, in order;
// list 1 (the half list) keeps only the edges that own their pair and list 2 (its
// complement) the others, each in the row ranges of its own partition.
// One launch builds all three (CTAs k ncta .. (k+1) ncta - 1 take list k), so
// the passes share the GPU.
// ---------------------------------------------------------------------------
struct CompactList {
    const int32_t* part;
    int32_t *crow, *ccol, *cidx, *ccount;   // cidx may be null (the list is not used for s_e)
    float* cdist;
};

__global__ void __launch_bounds__(512, 3) k_compact(const int32_t* __restrict__ row_ptr, int ncta,
                                                  const int32_t* __restrict__ erow, const int32_t* __restrict__ col,
                                                  const float4* __restrict__ pos4, Box box, float rc, long long cap,
                                                  const DevMeta* meta, CompactList full, CompactList half,
                                                  CompactList rev)
{
    pdl_trigger();
    pdl_wait();
    const int list = (int)blockIdx.x / ncta;      // 0: full, 1: half (owning edges), 2: complement
    const bool is_half = list == 1, is_rev = list == 2;
    const CompactList L = list == 0 ? full : (is_half ? half : rev);
    int32_t* __restrict__ crow = L.crow;
    int32_t* __restrict__ ccol = L.ccol;
    int32_t* __restrict__ cidx = L.cidx;
    int32_t* __restrict__ ccount = L.ccount;
    float* __restrict__ cdist = L.cdist;
    const int32_t* __restrict__ part = L.part;
    constexpr int CI = 4;             // consecutive edges per thread and pass
    __shared__ int wcount[32];
    __shared__ int total_s;
    const int c = (int)blockIdx.x - list * ncta;
    const int r0 = part[c], r1 = part[c + 1];
    if (meta->n_edges > cap || r0 >= r1) {
        if (threadIdx.x == 0) ccount[c] = 0;
        return;
    }
    const long long e0 = row_ptr[r0], e1 = row_ptr[r1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long base = e0;
    for (long long eb = e0; eb < e1; eb += (long long)CI * blockDim.x) {
        const long long ef = eb + (long long)CI * threadIdx.x;
        int ii[CI], jj[CI];
        float dd[CI];
        unsigned vmask = 0;
#pragma unroll
        for (int q = 0; q < CI; ++q) {
            ii[q] = 0;
            jj[q] = 0;
            if (ef + q < e1) {
                ii[q] = erow[ef + q];
                jj[q] = col[ef + q];
            }
        }
#pragma unroll
        for (int q = 0; q < CI; ++q) {
            if (ef + q < e1) {
                float3 v;
                const float d = edge_distance(pos4[ii[q]], pos4[jj[q]], box, v);
                dd[q] = d;
                if (d < rc && d > 0.f && (!is_half || owns_pair(ii[q], jj[q])) && (!is_rev || !owns_pair(ii[q], jj[q])))
                    vmask |= 1u << q;
            }
        }
        // block-wide exclusive scan of the per-thread counts, edge order kept
        const int cnt = __popc(vmask);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) wcount[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int nw = blockDim.x >> 5;
            const int v = lane < nw ? wcount[lane] : 0;
            int wi = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += t;
            }
            if (lane < nw) wcount[lane] = wi - v;
            if (lane == 31) total_s = wi;
        }
        __syncthreads();
        long long k = base + wcount[warp] + (incl - cnt);
#pragma unroll
        for (int q = 0; q < CI; ++q) {
            if ((vmask >> q) & 1u) {
                crow[k] = ii[q];
                ccol[k] = jj[q];
                if (cidx) cidx[k] = (int32_t)(ef + q);
                cdist[k] = dd[q];
                ++k;
            }
        }
        base += total_s;
        __syncthreads();
    }
    if (threadIdx.x == 0) ccount[c] = (int32_t)(base - e0);
}

// The full list of the step's edges inside the cutoff and, when forces follow, the
// half list of the pair-derivative launches and its complement (the dE/dh launches)
cudaError_t launch_compact(schnet_ctx* c, bool with_half)
{
    Workspace& w = c->ws;
    const CompactList full{w.part, w.crow, w.ccol, w.cidx, w.ccount, w.cdist};
    const CompactList half{w.part_h, w.crow_h, w.ccol_h, w.cidx_h, w.ccount_h, w.cdist_h};
    const CompactList rev{w.part_r, w.crow_r, w.ccol_r, nullptr, w.ccount_r, w.cdist_r};
    c->launches += 1;
    // 512 threads, three CTAs per SM: the three lists' 3 x ncta CTAs run as one wave (a cap of four
    // per SM would hold the pass to 32 registers, and it runs 9 % slower there)
    return launch_pdl(k_compact, c->ncta * (with_half ? 3 : 1), 512, 0, c->s, (const int32_t*)w.row_ptr,
                      (int)c->ncta, (const int32_t*)w.erow, (const int32_t*)w.col, (const float4*)w.pos4, c->box,
                      c->cfg.cutoff, (long long)c->cap, (const DevMeta*)w.meta, full, half, rev);
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
static MPArgs make_args(schnet_ctx* c, int layer)
{
    Workspace& w = c->ws;
    MPArgs a;
    a.cdist = w.cdist;
    a.crow = w.crow;
    a.ccol = w.ccol;
    a.cidx = w.cidx;
    a.ccount = w.ccount;
    a.row_ptr = w.row_ptr;
    a.part = w.part;
    a.meta = w.meta;
    a.cap = c->cap;
    a.rc = c->cfg.cutoff;
    a.inv_rc = 1.0f / c->cfg.cutoff;
    a.mu0 = c->mu0;
    a.dmu = c->dmu;
    a.K = c->K;
    a.ngc = (float)(-1.4426950408889634 / (2.0 * (double)c->cfg.rbf_sigma * (double)c->cfg.rbf_sigma));
    a.img = w.img + (size_t)layer * LAYER_IMG;
    a.s1 = w.s1 + layer * FP;
    a.s2 = w.s2 + layer * FP;
    a.b1 = w.b1 + layer * FP;
    a.b2 = w.b2 + layer * FP;
    a.h = w.h + (size_t)layer * c->N * FP;
    a.u = w.m;
    a.out = nullptr;
    a.s_edge = w.s_edge;
    a.accumulate_s = 0;
    return a;
}

template <int FMT, int NW, int NX>
static cudaError_t set_attrs()
{
    const int sf = (int)smem_bytes<TE_F, false>(), sb = (int)smem_bytes<TE_B, true>();
    cudaError_t e = cudaFuncSetAttribute(k_cfconv_fwd<FMT, NW, NX>, cudaFuncAttributeMaxDynamicSharedMemorySize, sf);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_cfconv_bwd<FMT, NW, NX, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, sb);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_cfconv_bwd<FMT, NW, NX, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, sb);
    return e;
}

cudaError_t cfconv_init_attributes()
{
    cudaError_t e;
    if ((e = set_attrs<0, 2, 2>()) != cudaSuccess) return e;
    if ((e = set_attrs<0, 1, 2>()) != cudaSuccess) return e;
    if ((e = set_attrs<1, 1, 2>()) != cudaSuccess) return e;
    return set_attrs<0, 1, 1>();
}

// operand formats: fp32 weights (fp16 hi+lo weights and activations), fp16 or bf16
// weights (one weight term, hi+lo activations), fp16 weights with fp16 activations
static cudaError_t launch_fwd(schnet_ctx* c, const MPArgs& a)
{
    const size_t sm = smem_bytes<TE_F, false>();
    if (c->n_xterms == 1)
        return launch_pdl(k_cfconv_fwd<0, 1, 1>, c->ncta, NT, sm, c->s, a);
    else if (c->weight_fmt == 0 && c->n_wterms == 2)
        return launch_pdl(k_cfconv_fwd<0, 2, 2>, c->ncta, NT, sm, c->s, a);
    else if (c->weight_fmt == 0)
        return launch_pdl(k_cfconv_fwd<0, 1, 2>, c->ncta, NT, sm, c->s, a);
    else
        return launch_pdl(k_cfconv_fwd<1, 1, 2>, c->ncta, NT, sm, c->s, a);
}

template <bool DH>
static cudaError_t launch_bwd(schnet_ctx* c, const MPArgs& a)
{
    const size_t sm = smem_bytes<TE_B, true>();
    if (c->n_xterms == 1)
        return launch_pdl(k_cfconv_bwd<0, 1, 1, DH>, c->ncta, NT, sm, c->s, a);
    else if (c->weight_fmt == 0 && c->n_wterms == 2)
        return launch_pdl(k_cfconv_bwd<0, 2, 2, DH>, c->ncta, NT, sm, c->s, a);
    else if (c->weight_fmt == 0)
        return launch_pdl(k_cfconv_bwd<0, 1, 2, DH>, c->ncta, NT, sm, c->s, a);
    else
        return launch_pdl(k_cfconv_bwd<1, 1, 2, DH>, c->ncta, NT, sm, c->s, a);
}

// m = sum_j h_j (.) W_ij of interaction `layer`
cudaError_t launch_cfconv_fwd(schnet_ctx* c, int layer)
{
    MPArgs a = make_args(c, layer);
    a.out = c->ws.m;
    c->launches += 1;
    return launch_fwd(c, a);
}

// The rest of dE/dh_i = sum_j u_j (.) W_ij with u = dE/dm of interaction `layer`:
// the terms over the complementary list, the edges that do not own their pair
// (the pair launch formed the half list's terms in dh), written to dh2 by the
// forward kernel's segment sum with u gathered in place of h; the atom-wise
// backward adds the two
cudaError_t launch_cfconv_dh(schnet_ctx* c, int layer)
{
    MPArgs a = make_args(c, layer);
    a.crow = c->ws.crow_r;
    a.ccol = c->ws.ccol_r;
    a.cdist = c->ws.cdist_r;
    a.ccount = c->ws.ccount_r;
    a.part = c->ws.part_r;
    a.h = c->ws.m;
    a.out = c->ws.dh2;
    c->launches += 1;
    return launch_fwd(c, a);
}

// Pair derivatives of interaction `layer` over the half list, written to s_e of
// each pair's owning edge (added to the later interactions' when accumulate_s);
// with_dh: also the half list's share of dE/dh (its edges' terms), written to dh
cudaError_t launch_cfconv_pair(schnet_ctx* c, int layer, int accumulate_s, bool with_dh)
{
    MPArgs a = make_args(c, layer);
    a.crow = c->ws.crow_h;
    a.ccol = c->ws.ccol_h;
    a.cidx = c->ws.cidx_h;
    a.cdist = c->ws.cdist_h;
    a.ccount = c->ws.ccount_h;
    a.part = c->ws.part_h;
    a.out = c->ws.dh;
    a.accumulate_s = accumulate_s;
    c->launches += 1;
    return with_dh ? launch_bwd<true>(c, a) : launch_bwd<false>(c, a);
}

}  // namespace schnet

// ---------------------------------------------------------------------------
// test tap: the FMA-pipe exponential on its own
// ---------------------------------------------------------------------------
namespace schnet {
__global__ void k_test_exp2(const float* __restrict__ x, float* __restrict__ y, long long n)
{
    const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float2 v = ex2_fma2(make_float2(x[i], i + 1 < n ? x[i + 1] : 0.0f));
    y[i] = v.x;
    if (i + 1 < n) y[i + 1] = v.y;
}
}  // namespace schnet

extern "C" schnet_status schnet_test_exp2(const float* d_x, float* d_y, int64_t n, void* cuda_stream)
{
    if (!d_x || !d_y || n < 0) return SCHNET_ERR_INVALID_ARG;
    if (n == 0) return SCHNET_OK;
    const long long pairs = (n + 1) / 2;
    schnet::k_test_exp2<<<(unsigned)((pairs + 255) / 256), 256, 0, (cudaStream_t)cuda_stream>>>(d_x, d_y, n);
    return cudaGetLastError() == cudaSuccess ? SCHNET_OK : SCHNET_ERR_CUDA;
}
