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
    const int32_t* erow;
    const int32_t* col;
    const int32_t* row_ptr;
    const int32_t* part;
    DevMeta* meta;
    long long cap;
    Box box;
    float rc, inv_rc;
    float mu0, dmu, inv2s2, invs2;
    int K;
    const uint8_t* img;   // this layer's packed W1^T / W2^T images
    const float *s1, *s2, *b1, *b2;  // this layer's scales and biases [FP]
    const float* h;       // [N][FP]
    const float* u;       // [N][FP]   (backward)
    float* out;           // m (forward) or dh (backward)   [N][FP]
    float* s_edge;        // [cap]     (backward)
    int accumulate_s;
};

// shared-memory map (bytes)
constexpr uint32_t SM_W1 = 0;                          // W1^T hi, lo   2 x 16 KB
constexpr uint32_t SM_W2 = 32768;                      // W2^T hi, lo   2 x 32 KB
constexpr uint32_t SM_X = 98304;                       // fwd: rbf hi/lo (32 KB) ; bwd: rbf, rbf' then a (64 KB)
constexpr uint32_t SM_FWD_A = 131072;                  // fwd: a hi/lo (64 KB)
constexpr uint32_t SM_BWD_Y = 163840;                  // bwd: ssp'(p) p' hi/lo (64 KB)
constexpr uint32_t SM_META_FWD = 196608;
constexpr uint32_t SM_META_BWD = 229376;
constexpr uint32_t META_BYTES = 2048 + 16;
constexpr uint32_t SMEM_FWD = SM_META_FWD + META_BYTES;
constexpr uint32_t SMEM_BWD = SM_META_BWD + META_BYTES;

constexpr uint32_t RBF_TERM = TILE_E * KP * 2;   // 16 KB: one 16-bit term of a [128 x 64] tile
constexpr uint32_t ACT_TERM = TILE_E * FP * 2;   // 32 KB: one 16-bit term of a [128 x 128] tile
constexpr uint32_t WAIT_POLLS = 1u << 22;

struct TileMeta {
    int32_t row[TILE_E];
    int32_t col[TILE_E];   // -1: padding or d >= r_c (masked)
    float fc[TILE_E];
    float dfc[TILE_E];
};

__device__ __forceinline__ void copy_weights(uint8_t* smem, const uint8_t* __restrict__ img)
{
    const uint4* src = reinterpret_cast<const uint4*>(img);
    uint4* dst = reinterpret_cast<uint4*>(smem + SM_W1);
    for (int i = threadIdx.x; i < (int)(LAYER_IMG / 16); i += blockDim.x) dst[i] = __ldg(src + i);
}

__device__ __forceinline__ uint4 pack8(const uint16_t (&v)[8])
{
    return make_uint4((uint32_t)v[0] | ((uint32_t)v[1] << 16), (uint32_t)v[2] | ((uint32_t)v[3] << 16),
                      (uint32_t)v[4] | ((uint32_t)v[5] << 16), (uint32_t)v[6] | ((uint32_t)v[7] << 16));
}

// Stage R: thread t handles edge t of the tile: distance (minimum image),
// cutoff mask, Gaussian expansion (and its d-derivative when BWD) written as
// hi/lo 16-bit K-major B operands.
template <int FMT, bool BWD>
__device__ __forceinline__ void stage_rbf(const MPArgs& a, uint8_t* smem, TileMeta* tm, long long e0, int ne)
{
    const int t = threadIdx.x;
    float d = 0.f;
    bool valid = false;
    int i = 0, j = -1;
    if (t < ne) {
        long long e = e0 + t;
        i = a.erow[e];
        j = a.col[e];
        float4 pi = a.pos4[i], pj = a.pos4[j];
        float3 v = min_image(make_float3(pj.x - pi.x, pj.y - pi.y, pj.z - pi.z), a.box);
        d = sqrtf(v.x * v.x + v.y * v.y + v.z * v.z);
        valid = d < a.rc && d > 0.f;
    }
    float fc = 0.f, dfc = 0.f;
    if (valid) {
        float s, c;
        sincospif(d * a.inv_rc, &s, &c);
        fc = 0.5f * (c + 1.0f);
        dfc = -0.5f * 3.14159265358979f * a.inv_rc * s;
    }
    tm->row[t] = t < ne ? i : 0x7fffffff;
    tm->col[t] = valid ? j : -1;
    tm->fc[t] = fc;
    tm->dfc[t] = dfc;

    uint8_t* b_hi = smem + SM_X;
    uint8_t* b_lo = b_hi + RBF_TERM;
    uint8_t* p_hi = smem + SM_X + 2 * RBF_TERM;   // derivative tile (backward)
    uint8_t* p_lo = p_hi + RBF_TERM;
#pragma unroll
    for (int kg = 0; kg < KP / 8; ++kg) {
        uint16_t hi[8], lo[8], dhi[8], dlo[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            int k = kg * 8 + q;
            float g = 0.f, dg = 0.f;
            if (valid && k < a.K) {
                float x = d - (a.mu0 + (float)k * a.dmu);
                g = __expf(-x * x * a.inv2s2);
                dg = -x * a.invs2 * g;
            }
            Split<FMT>::run(g, hi[q], lo[q]);
            if (BWD) Split<FMT>::run(dg, dhi[q], dlo[q]);
        }
        uint32_t off = kmajor_off(t, kg * 8, TILE_E);
        *reinterpret_cast<uint4*>(b_hi + off) = pack8(hi);
        *reinterpret_cast<uint4*>(b_lo + off) = pack8(lo);
        if (BWD) {
            *reinterpret_cast<uint4*>(p_hi + off) = pack8(dhi);
            *reinterpret_cast<uint4*>(p_lo + off) = pack8(dlo);
        }
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
    bool ok = mbar_wait_bounded(bar, phase, WAIT_POLLS);
    phase ^= 1u;
    int bad = __syncthreads_or(!ok);
    if (bad) {
        if (threadIdx.x == 0) set_flag(meta, SCHNET_FLAG_TIMEOUT);
        return false;
    }
    tc_fence_after();
    return true;
}

// Write a 128-edge activation row (thread = feature f = K index) into an
// MN-major B operand: 8 consecutive edges per 16-byte store.
template <int FMT>
__device__ __forceinline__ void store_act_group(uint8_t* base, int f, int e8, const float* v)
{
    uint16_t hi[8], lo[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) Split<FMT>::run(v[q], hi[q], lo[q]);
    uint32_t off = mnmajor_off(e8, f, TILE_E);
    *reinterpret_cast<uint4*>(base + off) = pack8(hi);
    *reinterpret_cast<uint4*>(base + ACT_TERM + off) = pack8(lo);
}

// ---------------------------------------------------------------------------
// forward: m_i = sum_j h_j (.) W(d_ij)
// ---------------------------------------------------------------------------
template <int FMT, int NW>
__global__ void __launch_bounds__(128, 1) k_cfconv_fwd(MPArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    TileMeta* tm = reinterpret_cast<TileMeta*>(smem + SM_META_FWD);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + SM_META_FWD + 2048);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + SM_META_FWD + 2056);

    if (a.meta->n_edges > a.cap) return;
    const int r0 = a.part[blockIdx.x], r1 = a.part[blockIdx.x + 1];
    if (r0 >= r1) return;
    const long long e0 = a.row_ptr[r0], e1 = a.row_ptr[r1];
    const int f = threadIdx.x, warp = threadIdx.x >> 5;

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
    const uint32_t tP = tmem, tQ = tmem + 128;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t id = idesc_f16(128, TILE_E, FMT, 0);
    const uint32_t id_mn = idesc_f16(128, TILE_E, FMT, 1);

    const float s1 = a.s1[f], b1 = a.b1[f], s2 = a.s2[f], b2 = a.b2[f];
    int cur = r0;
    float acc = 0.f;
    uint32_t phase = 0;
    bool ok = true;

    for (long long t0 = e0; t0 < e1 && ok; t0 += TILE_E) {
        const int ne = (int)min((long long)TILE_E, e1 - t0);
        stage_rbf<FMT, false>(a, smem, tm, t0, ne);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            issue_gemm<NW>(tP, sbase + SM_W1, (uint32_t)W1_IMG, sbase + SM_X, RBF_TERM, KP / 16, id);
            mma_commit(bar);
        }
        if (!(ok = wait_mma(bar, phase, a.meta))) break;

        // epilogue 1: a = ssp(s1 P + b1) -> MN-major B operand of GEMM2
#pragma unroll 1
        for (int c = 0; c < TILE_E / 32; ++c) {
            float r[32];
            tmem_ld32(tP + lane_off + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) r[q] = ssp(fmaf(s1, r[q], b1));
#pragma unroll
            for (int g = 0; g < 4; ++g) store_act_group<FMT>(smem + SM_FWD_A, f, c * 32 + g * 8, r + g * 8);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            issue_gemm<NW>(tQ, sbase + SM_W2, (uint32_t)W2_IMG, sbase + SM_FWD_A, ACT_TERM, FP / 16, id_mn);
            mma_commit(bar);
        }
        if (!(ok = wait_mma(bar, phase, a.meta))) break;

        // epilogue 2: W = f_c (s2 Q + b2); segment sum of h_j (.) W per row
#pragma unroll 1
        for (int c = 0; c < TILE_E / 32; ++c) {
            if (c * 32 >= ne) break;
            float r[32];
            tmem_ld32(tQ + lane_off + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const int e = c * 32 + q;
                if (e >= ne) break;
                const int row = tm->row[e];
                if (row != cur) {
                    a.out[(size_t)cur * FP + f] = acc;
                    for (int rr = cur + 1; rr < row; ++rr) a.out[(size_t)rr * FP + f] = 0.f;
                    cur = row;
                    acc = 0.f;
                }
                const int j = tm->col[e];
                if (j >= 0) {
                    float w = tm->fc[e] * fmaf(s2, r[q], b2);
                    acc = fmaf(w, __ldg(a.h + (size_t)j * FP + f), acc);
                }
            }
        }
        tc_fence_before();
        __syncthreads();   // tile metadata and operand tiles are rewritten next
    }

    if (ok) {
        a.out[(size_t)cur * FP + f] = acc;
        for (int rr = cur + 1; rr < r1; ++rr) a.out[(size_t)rr * FP + f] = 0.f;
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
template <int FMT, int NW>
__global__ void __launch_bounds__(128, 1) k_cfconv_bwd(MPArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    TileMeta* tm = reinterpret_cast<TileMeta*>(smem + SM_META_BWD);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + SM_META_BWD + 2048);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + SM_META_BWD + 2056);
    float* partial = reinterpret_cast<float*>(smem + SM_BWD_Y);   // [4][128] after GEMM2

    if (a.meta->n_edges > a.cap) return;
    const int r0 = a.part[blockIdx.x], r1 = a.part[blockIdx.x + 1];
    if (r0 >= r1) return;
    const long long e0 = a.row_ptr[r0], e1 = a.row_ptr[r1];
    const int f = threadIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

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
    const uint32_t tP = tmem, tPd = tmem + 128, tQ = tmem + 256, tQd = tmem + 384;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t id = idesc_f16(128, TILE_E, FMT, 0);
    const uint32_t id_mn = idesc_f16(128, TILE_E, FMT, 1);

    const float s1 = a.s1[f], b1 = a.b1[f], s2 = a.s2[f], b2 = a.b2[f];
    int cur = r0;
    float acc = 0.f;
    float u_row = a.u[(size_t)r0 * FP + f];
    uint32_t phase = 0;
    bool ok = true;

    for (long long t0 = e0; t0 < e1 && ok; t0 += TILE_E) {
        const int ne = (int)min((long long)TILE_E, e1 - t0);
        stage_rbf<FMT, true>(a, smem, tm, t0, ne);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            issue_gemm<NW>(tP, sbase + SM_W1, (uint32_t)W1_IMG, sbase + SM_X, RBF_TERM, KP / 16, id);
            issue_gemm<NW>(tPd, sbase + SM_W1, (uint32_t)W1_IMG, sbase + SM_X + 2 * RBF_TERM, RBF_TERM, KP / 16,
                           id);
            mma_commit(bar);
        }
        if (!(ok = wait_mma(bar, phase, a.meta))) break;

        // epilogue 1: a = ssp(p), b = ssp'(p) p'   (p = s1 P + b1, p' = s1 P')
#pragma unroll 1
        for (int c = 0; c < TILE_E / 32; ++c) {
            float r[32], rd[32];
            tmem_ld32(tP + lane_off + c * 32, r);
            tmem_ld32(tPd + lane_off + c * 32, rd);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                float sv, gv;
                ssp_and_grad(fmaf(s1, r[q], b1), sv, gv);
                r[q] = sv;
                rd[q] = gv * s1 * rd[q];
            }
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                store_act_group<FMT>(smem + SM_X, f, c * 32 + g * 8, r + g * 8);
                store_act_group<FMT>(smem + SM_BWD_Y, f, c * 32 + g * 8, rd + g * 8);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            issue_gemm<NW>(tQ, sbase + SM_W2, (uint32_t)W2_IMG, sbase + SM_X, ACT_TERM, FP / 16, id_mn);
            issue_gemm<NW>(tQd, sbase + SM_W2, (uint32_t)W2_IMG, sbase + SM_BWD_Y, ACT_TERM, FP / 16, id_mn);
            mma_commit(bar);
        }
        if (!(ok = wait_mma(bar, phase, a.meta))) break;

        // epilogue 2: W = f_c z, W' = f_c' z + f_c z'  (z = s2 Q + b2, z' = s2 Q')
#pragma unroll 1
        for (int c = 0; c < TILE_E / 32; ++c) {
            float r[32], rd[32];
            tmem_ld32(tQ + lane_off + c * 32, r);
            tmem_ld32(tQd + lane_off + c * 32, rd);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const int e = c * 32 + q;
                float tval = 0.f;
                if (e < ne) {
                    const int row = tm->row[e];
                    if (row != cur) {
                        a.out[(size_t)cur * FP + f] = acc;
                        for (int rr = cur + 1; rr < row; ++rr) a.out[(size_t)rr * FP + f] = 0.f;
                        cur = row;
                        acc = 0.f;
                        u_row = a.u[(size_t)row * FP + f];
                    }
                    const int j = tm->col[e];
                    if (j >= 0) {
                        const float z = fmaf(s2, r[q], b2);
                        const float fcv = tm->fc[e];
                        const float w = fcv * z;
                        const float wd = fmaf(tm->dfc[e], z, fcv * s2 * rd[q]);
                        const float uj = __ldg(a.u + (size_t)j * FP + f);
                        const float hj = __ldg(a.h + (size_t)j * FP + f);
                        acc = fmaf(w, uj, acc);
                        tval = wd * u_row * hj;
                    }
                }
                rd[q] = tval;
            }
            // transpose-reduce the 32 per-edge values over the warp's 32 features:
            // afterwards lane l holds the warp's sum for edge c*32 + l.
#pragma unroll
            for (int sh = 16; sh >= 1; sh >>= 1) {
                const bool upper = (lane & sh) != 0;
#pragma unroll
                for (int k = 0; k < sh; ++k) {
                    float send = upper ? rd[k] : rd[k + sh];
                    float keep = upper ? rd[k + sh] : rd[k];
                    rd[k] = keep + __shfl_xor_sync(0xffffffffu, send, sh);
                }
            }
            partial[warp * TILE_E + c * 32 + lane] = rd[0];
        }
        __syncthreads();
        if (f < ne) {
            float s = partial[f] + partial[TILE_E + f] + partial[2 * TILE_E + f] + partial[3 * TILE_E + f];
            float* dst = a.s_edge + (t0 + f);
            *dst = a.accumulate_s ? *dst + s : s;
        }
        tc_fence_before();
        __syncthreads();
    }

    if (ok) {
        a.out[(size_t)cur * FP + f] = acc;
        for (int rr = cur + 1; rr < r1; ++rr) a.out[(size_t)rr * FP + f] = 0.f;
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
// launchers
// ---------------------------------------------------------------------------
static MPArgs make_args(schnet_ctx* c, int layer)
{
    Workspace& w = c->ws;
    MPArgs a;
    a.pos4 = w.pos4;
    a.erow = w.erow;
    a.col = w.col;
    a.row_ptr = w.row_ptr;
    a.part = w.part;
    a.meta = w.meta;
    a.cap = c->cap;
    a.box = c->box;
    a.rc = c->cfg.cutoff;
    a.inv_rc = 1.0f / c->cfg.cutoff;
    a.mu0 = c->mu0;
    a.dmu = c->dmu;
    a.inv2s2 = 1.0f / (2.0f * c->cfg.rbf_sigma * c->cfg.rbf_sigma);
    a.invs2 = 1.0f / (c->cfg.rbf_sigma * c->cfg.rbf_sigma);
    a.K = c->K;
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
        k_cfconv_fwd<0, 2><<<c->ncta, 128, SMEM_FWD, c->s>>>(a);
    else if (c->weight_fmt == 0)
        k_cfconv_fwd<0, 1><<<c->ncta, 128, SMEM_FWD, c->s>>>(a);
    else
        k_cfconv_fwd<1, 1><<<c->ncta, 128, SMEM_FWD, c->s>>>(a);
    c->launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_cfconv_bwd(schnet_ctx* c, int layer, int accumulate_s)
{
    MPArgs a = make_args(c, layer);
    a.out = c->ws.dh;
    a.accumulate_s = accumulate_s;
    if (c->weight_fmt == 0 && c->n_wterms == 2)
        k_cfconv_bwd<0, 2><<<c->ncta, 128, SMEM_BWD, c->s>>>(a);
    else if (c->weight_fmt == 0)
        k_cfconv_bwd<0, 1><<<c->ncta, 128, SMEM_BWD, c->s>>>(a);
    else
        k_cfconv_bwd<1, 1><<<c->ncta, 128, SMEM_BWD, c->s>>>(a);
    c->launches += 1;
    return cudaGetLastError();
}

}  // namespace schnet
