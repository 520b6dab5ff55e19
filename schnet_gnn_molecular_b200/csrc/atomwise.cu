// Atom-wise parts of SchNet: the embedding (a per-type table gather), and on the
// sm_100a tensor cores the interaction's in/out dense layers with the residual
// update, the per-atom readout and their backward pass; the per-replica sums.
//
// Model reading (FlashSchNet paper-curation summary, How / Figure 2 caption:
// positions and embeddings pass through interaction blocks; readout per atom
// summed to the energy): h = x W_in; x += ssp(m Wo1 + bo1) Wo2 + bo2;
// eps = ssp(x R1 + c1) R2 + c2.  Backward (chain rule, by hand):
//   g^L = (ssp'(pr) (.) R2) R1^T;  u = ((g Wo2^T) (.) ssp'(q)) Wo1^T;
//   g^l = g^{l+1} + dh W_in^T.
//
// Each launch is a persistent kernel over tiles of 128 atoms that chains up to
// three dense layers.  Every layer is one transposed GEMM on tcgen05,
// D[o][atom] = A[o][k] X[atom][k]: the weights A (one output channel per lane,
// channel-scaled, hi/lo 16-bit terms) sit in TMEM for the whole launch, the
// activations X are staged in shared memory as hi/lo 16-bit terms after a
// power-of-two scaling of the whole tile (so small gradients keep their
// relative precision), and the accumulator D (128 TMEM columns) is read back
// one feature per thread, 32 atoms per thread, for the elementwise epilogue.
// 3 MMAs per K-step (hi*hi + lo_w*hi + hi*lo_x), fp32 accumulation.
#include <algorithm>

#include "internal.h"

namespace schnet {

constexpr int AWT = 512;                      // 16 warps: TMEM lane quadrant = warp % 4, atom chunk = warp / 4
constexpr int ATILE = 128;                    // atoms per tile (GEMM N)
constexpr uint32_t AW_BTERM = ATILE * FP * 2; // 32 KB: one 16-bit term of the [128 atoms x 128] B tile
constexpr uint32_t AW_SMEM = 2 * AW_BTERM + 128 + 64;   // B hi/lo, per-warp maxima, mbarrier + TMEM slot
constexpr uint32_t AW_POLLS = 1u << 22;
constexpr uint32_t AW_ACC = 0;                // TMEM columns 0..127: accumulator
constexpr uint32_t AW_SLOT = 128;             // TMEM columns 128 + 128 s: weight slot s (hi 64, lo 64)

enum { AW_FWD = 1, AW_TOP = 2, AW_BWD = 3 };

struct AWArgs {
    int N, ntiles;
    int ngemm;                    // dense layers chained in this launch (1..3)
    int last;                     // AW_FWD: readout instead of the next layer's h
    const uint8_t* img[3];        // the layers' packed A images (hi term, then lo term)
    const float* sc[3];           // their per-row scales [FP]
    const float *bo1, *bo2, *c1, *R2, *c2;
    float *x, *h_out, *q, *m, *g, *pr, *eps;
    const float *dh, *dh2;        // backward: dE/dh as two parts (half list, complement) that add up
    const float* q_in;            // backward: q of the layer whose u is formed
    DevMeta* meta;
};

// per-tile power-of-two scale: maps the tile's largest |value| into [2^14, 2^15)
__device__ __forceinline__ float tile_scale(const float (&v)[32], float* wmax, float& inv)
{
    float mx = 0.f;
#pragma unroll
    for (int q = 0; q < 32; ++q) mx = fmaxf(mx, fabsf(v[q]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    __syncthreads();                                  // previous readers of wmax are done
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = 0.f;
#pragma unroll
    for (int w = 0; w < AWT / 32; ++w) mx = fmaxf(mx, wmax[w]);
    int e = 0;
    const int ex = (int)((__float_as_uint(mx) >> 23) & 255u);
    if (ex > 0 && ex < 255) e = 14 - (ex - 127);      // 2^(ex-127) <= mx < 2^(ex-126)
    e = max(-120, min(120, e));
    inv = __uint_as_float((uint32_t)(127 - e) << 23);
    return __uint_as_float((uint32_t)(127 + e) << 23);
}

// stage 32 values (feature f = K index, atoms 32c .. 32c+31 = B rows) as hi/lo MN-major B
__device__ __forceinline__ void stage_b(uint8_t* B, const float (&v)[32], float s, int c, int f)
{
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        float w[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) w[q] = v[g * 8 + q] * s;
        store8<0>(B, B + AW_BTERM, mnmajor_off(c * 32 + g * 8, f, ATILE), w);
    }
}

// one layer: D = A_slot * B^T, then the accumulator row of this thread (32 atoms)
__device__ __forceinline__ bool aw_gemm(uint32_t tmem, int slot, uint32_t sB, uint64_t* bar, uint32_t& phase,
                                        DevMeta* meta, uint32_t tD, float (&d)[32])
{
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
        tc_fence_after();
        const uint32_t id = idesc_f16(128, ATILE, 0, 1);
        const uint32_t ahi = tmem + AW_SLOT + 128 * slot, alo = ahi + 64;
        const uint64_t bh0 = smem_desc(sB, ATILE * 16, 128), bl0 = smem_desc(sB + AW_BTERM, ATILE * 16, 128);
        // the two small correction products first, the hi x hi product last: the tensor
        // core's fp32 accumulation does not round to nearest, so every MMA added to an
        // accumulator that already holds the large sum costs a little accuracy
#pragma unroll
        for (int ks = 0; ks < FP / 16; ++ks) {
            const uint64_t step = (uint64_t)((ks * 2 * ATILE * 16) >> 4);   // start-address field only
            mma_f16_ts(tmem + AW_ACC, alo + ks * 8, bh0 + step, id, ks > 0 ? 1u : 0u);
            mma_f16_ts(tmem + AW_ACC, ahi + ks * 8, bl0 + step, id, 1u);
        }
#pragma unroll
        for (int ks = 0; ks < FP / 16; ++ks) {
            const uint64_t step = (uint64_t)((ks * 2 * ATILE * 16) >> 4);
            mma_f16_ts(tmem + AW_ACC, ahi + ks * 8, bh0 + step, id, 1u);
        }
        mma_commit(bar);
    }
    bool ok = true;
    if ((threadIdx.x >> 5) == 0) ok = mbar_wait_bounded(bar, phase, AW_POLLS);
    if (__syncthreads_or(!ok)) {
        if (threadIdx.x == 0) set_flag(meta, SCHNET_FLAG_TIMEOUT);
        return false;
    }
    phase ^= 1u;
    tc_fence_after();
    tmem_ld32(tD, d);
    tmem_ld_wait();
    return true;
}

template <int MODE>
__global__ void __launch_bounds__(AWT, 1) k_atomwise(AWArgs a)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    uint8_t* B = sm;
    float* wmax = reinterpret_cast<float*>(sm + 2 * AW_BTERM);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 2 * AW_BTERM + 128);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qd = warp & 3, c = warp >> 2;
    const int f = qd * 32 + lane;                    // this thread's feature (output row / next K index)

    pdl_trigger();
    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
    // weights: warp c of quadrant qd loads (term c >> 1, half c & 1) of every slot, all slots'
    // rows first (one trip to L2), then the TMEM stores
    {
        uint32_t x[3][32];
#pragma unroll
        for (int s = 0; s < 3; ++s) {
            if (s >= a.ngemm) break;
            weight_row(a.img[s] + (c >> 1) * AW_BTERM, f, c & 1, x[s]);
        }
#pragma unroll
        for (int s = 0; s < 3; ++s) {
            if (s >= a.ngemm) break;
            tmem_st32(lane_base + AW_SLOT + 128 * s + (c >> 1) * 64 + (c & 1) * 32, x[s]);
        }
    }
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    const uint32_t sB = smem_u32(B);
    const uint32_t tD = lane_base + AW_ACC + c * 32;
    float sc[3];
#pragma unroll
    for (int s = 0; s < 3; ++s) sc[s] = s < a.ngemm ? a.sc[s][f] : 0.f;
    pdl_wait();                                      // the previous kernel's results from here on
    uint32_t phase = 0;
    bool ok = true;

    for (int tile = blockIdx.x; tile < a.ntiles && ok; tile += gridDim.x) {
        const int i0 = tile * ATILE + c * 32;       // this thread's first atom
        float v[32], d[32];
        float s, inv;
        auto row_ok = [&](int q) { return i0 + q < a.N; };
        auto at = [&](int q, int w) { return (size_t)(i0 + q) * w + f; };
        // ---- input of the first layer
        if (MODE == AW_FWD) {
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] = row_ok(q) ? __ldg(a.m + at(q, FP)) : 0.f;
        } else if (MODE == AW_TOP) {
            // y = ssp'(pr) (.) R2 over the readout's hidden units (K = HP, zero beyond)
            const float r2 = f < HP ? __ldg(a.R2 + f) : 0.f;
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] = (f < HP && row_ok(q)) ? sigmoidf(__ldg(a.pr + at(q, HP))) * r2 : 0.f;
        } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] = row_ok(q) ? __ldg(a.dh + at(q, FP)) + __ldg(a.dh2 + at(q, FP)) : 0.f;
        }
        s = tile_scale(v, wmax, inv);
        stage_b(B, v, s, c, f);
        if (!(ok = aw_gemm(tmem, 0, sB, bar, phase, a.meta, tD, d))) break;
        const float k0 = sc[0] * inv;
        if (MODE == AW_FWD) {
            // q = m Wo1 + bo1 ; a = ssp(q)
            const float b = __ldg(a.bo1 + f);
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const float qv = fmaf(d[q], k0, b);
                if (row_ok(q)) a.q[at(q, FP)] = qv;
                v[q] = ssp(qv);
            }
        } else if (MODE == AW_TOP) {
            // g = y R1^T
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                v[q] = d[q] * k0;
                if (row_ok(q)) a.g[at(q, FP)] = v[q];
            }
        } else {
            // g += dh W_in^T
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                v[q] = row_ok(q) ? fmaf(d[q], k0, __ldg(a.g + at(q, FP))) : 0.f;
                if (row_ok(q)) a.g[at(q, FP)] = v[q];
            }
        }
        if (a.ngemm < 2) continue;
        // ---- second layer
        s = tile_scale(v, wmax, inv);
        stage_b(B, v, s, c, f);
        if (!(ok = aw_gemm(tmem, 1, sB, bar, phase, a.meta, tD, d))) break;
        const float k1 = sc[1] * inv;
        if (MODE == AW_FWD) {
            // x += a Wo2 + bo2
            const float b = __ldg(a.bo2 + f);
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                float xv = 0.f;
                if (row_ok(q)) {
                    xv = a.x[at(q, FP)] + fmaf(d[q], k1, b);
                    a.x[at(q, FP)] = xv;
                }
                v[q] = xv;
            }
        } else {
            // t = (g Wo2^T) (.) ssp'(q)
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] = row_ok(q) ? d[q] * k1 * sigmoidf(__ldg(a.q_in + at(q, FP))) : 0.f;
        }
        // ---- third layer
        s = tile_scale(v, wmax, inv);
        stage_b(B, v, s, c, f);
        if (!(ok = aw_gemm(tmem, 2, sB, bar, phase, a.meta, tD, d))) break;
        const float k2 = sc[2] * inv;
        if (MODE == AW_FWD && !a.last) {
#pragma unroll
            for (int q = 0; q < 32; ++q)
                if (row_ok(q)) a.h_out[at(q, FP)] = d[q] * k2;
        } else if (MODE == AW_FWD) {
            // readout: pr = x R1 + c1 (rows f < HP); eps = sum_k ssp(pr_k) R2_k + c2, summed over
            // the hidden units through shared memory (B is dead after the last GEMM)
            float* S = reinterpret_cast<float*>(B);      // [HP][ATILE + 1]
            if (f < HP) {
                const float cb = __ldg(a.c1 + f), r2 = __ldg(a.R2 + f);
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const float p = fmaf(d[q], k2, cb);
                    if (row_ok(q)) a.pr[at(q, HP)] = p;
                    S[f * (ATILE + 1) + c * 32 + q] = ssp(p) * r2;
                }
            }
            __syncthreads();
            if (threadIdx.x < ATILE) {
                const int i = tile * ATILE + threadIdx.x;
                float e = 0.f;
                for (int k = 0; k < HP; ++k) e += S[k * (ATILE + 1) + threadIdx.x];
                if (i < a.N) a.eps[i] = e + __ldg(a.c2);
            }
        } else {
            // u = t Wo1^T, into m
#pragma unroll
            for (int q = 0; q < 32; ++q)
                if (row_ok(q)) a.m[at(q, FP)] = d[q] * k2;
        }
    }
    // error exit: give an MMA still in flight a bounded chance to retire before freeing TMEM
    if (!ok && threadIdx.x == 0) mbar_wait_bounded(bar, phase, AW_POLLS);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// per-replica sums (float64 accumulation, fixed order)
// ---------------------------------------------------------------------------
__global__ void k_chunk_sums(const float* __restrict__ v, const int32_t* __restrict__ lo,
                             const int32_t* __restrict__ hi, double* __restrict__ partial)
{
    pdl_trigger();
    pdl_wait();
    int c = blockIdx.x;
    double s = 0.0;
    for (int i = lo[c] + threadIdx.x; i < hi[c]; i += blockDim.x) s += (double)v[i];
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    __shared__ double ws[32];
    if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += ws[w];
        partial[c] = t;
    }
}

__global__ void k_replica_sums(int R, const int32_t* __restrict__ chunk_rep, int nchunk,
                               const double* __restrict__ partial, double* __restrict__ out, DevMeta* meta)
{
    pdl_trigger();
    pdl_wait();
    int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= R) return;
    // chunks of replica r are contiguous; find them by scanning the (small) table
    double s = 0.0;
    for (int c = 0; c < nchunk; ++c)
        if (chunk_rep[c] == r) s += partial[c];
    out[r] = s;
    if (!isfinite(s)) set_flag(meta, SCHNET_FLAG_NONFINITE);
}

// images and scales of the atom-wise layers: per layer l, matrix id 6 l + j with
// j = 0 Wo1^T, 1 Wo2^T, 2 W_in^T (forward), 3 W_in, 4 Wo2, 5 Wo1 (backward);
// then 6 L = R1^T (readout), 6 L + 1 = R1 (readout backward)
static AWArgs aw_args(schnet_ctx* c, int mode, int layer)
{
    Workspace& w = c->ws;
    const int L = c->L;
    AWArgs a{};
    a.N = c->N;
    a.ntiles = (c->N + ATILE - 1) / ATILE;
    a.bo1 = w.bo1 + layer * FP; a.bo2 = w.bo2 + layer * FP;
    a.c1 = w.c1; a.R2 = w.R2; a.c2 = w.c2;
    a.x = w.x; a.q = w.q + (size_t)layer * c->N * FP; a.m = w.m; a.g = w.g; a.dh = w.dh; a.dh2 = w.dh2; a.pr = w.pr;
    a.eps = w.eps; a.meta = w.meta;
    int ids[3] = {0, 0, 0};
    if (mode == AW_FWD) {
        a.ngemm = 3; ids[0] = 6 * layer; ids[1] = 6 * layer + 1;
        a.last = layer + 1 == L;
        ids[2] = a.last ? 6 * L : 6 * (layer + 1) + 2;
        a.h_out = a.last ? nullptr : w.h + (size_t)(layer + 1) * c->N * FP;
    } else if (mode == AW_TOP) {
        a.ngemm = 3; ids[0] = 6 * L + 1; ids[1] = 6 * (L - 1) + 4; ids[2] = 6 * (L - 1) + 5;
        a.q_in = w.q + (size_t)(L - 1) * c->N * FP;
    } else {
        a.ngemm = layer > 0 ? 3 : 1;
        ids[0] = 6 * layer + 3;
        if (layer > 0) {
            ids[1] = 6 * (layer - 1) + 4; ids[2] = 6 * (layer - 1) + 5;
            a.q_in = w.q + (size_t)(layer - 1) * c->N * FP;
        }
    }
    for (int s = 0; s < 3; ++s) {
        a.img[s] = w.aw_img + (size_t)ids[s] * AW_IMG;
        a.sc[s] = w.aw_sc + (size_t)ids[s] * FP;
    }
    return a;
}

cudaError_t atomwise_init_attributes()
{
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k_atomwise<AW_FWD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)AW_SMEM)))
        return e;
    if ((e = cudaFuncSetAttribute(k_atomwise<AW_TOP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)AW_SMEM)))
        return e;
    return cudaFuncSetAttribute(k_atomwise<AW_BWD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)AW_SMEM);
}

static int aw_grid(schnet_ctx* c) { return std::min((c->N + ATILE - 1) / ATILE, c->nsm); }

// Embedding and the first h: one warp per slot, four features per lane.  x0 = emb[z]
// and h0 = (emb W_in)[z] are rows of per-type tables (the second formed on the host
// in float64), so no GEMM is needed for interaction 0's input.
__global__ void k_embed(int n, int T, const int32_t* __restrict__ types, const int32_t* __restrict__ perm,
                        const float4* __restrict__ emb, const float4* __restrict__ emb_h0, float4* __restrict__ x,
                        float4* __restrict__ h, DevMeta* meta)
{
    pdl_trigger();
    pdl_wait();
    const int k = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (k >= n) return;
    int z = __ldg(types + __ldg(perm + k));
    if (z < 0 || z >= T) {
        if (lane == 0) set_flag(meta, SCHNET_FLAG_BADTYPE);
        z = 0;
    }
    x[(size_t)k * (FP / 4) + lane] = __ldg(emb + (size_t)z * (FP / 4) + lane);
    h[(size_t)k * (FP / 4) + lane] = __ldg(emb_h0 + (size_t)z * (FP / 4) + lane);
}

cudaError_t launch_embed(schnet_ctx* c, const int32_t* types)
{
    Workspace& w = c->ws;
    static_assert(FP == 128, "one float4 per lane covers a padded feature row");
    const long long threads = (long long)c->N * 32;
    c->launches += 1;
    return launch_pdl(k_embed, (unsigned)((threads + 255) / 256), 256, 0, c->s, c->N, c->T, types,
                      (const int32_t*)w.perm, reinterpret_cast<const float4*>(w.emb),
                      reinterpret_cast<const float4*>(w.emb_h0), reinterpret_cast<float4*>(w.x),
                      reinterpret_cast<float4*>(w.h), w.meta);
}

cudaError_t launch_aw_fwd(schnet_ctx* c, int layer)
{
    c->launches += 1;
    return launch_pdl(k_atomwise<AW_FWD>, aw_grid(c), AWT, AW_SMEM, c->s, aw_args(c, AW_FWD, layer));
}

cudaError_t launch_aw_bwd_top(schnet_ctx* c)
{
    c->launches += 1;
    return launch_pdl(k_atomwise<AW_TOP>, aw_grid(c), AWT, AW_SMEM, c->s, aw_args(c, AW_TOP, c->L - 1));
}

cudaError_t launch_aw_bwd(schnet_ctx* c, int layer)
{
    c->launches += 1;
    return launch_pdl(k_atomwise<AW_BWD>, aw_grid(c), AWT, AW_SMEM, c->s, aw_args(c, AW_BWD, layer));
}

cudaError_t launch_replica_sum(schnet_ctx* c, const float* v, double* out)
{
    Workspace& w = c->ws;
    c->launches += 2;
    cudaError_t e = launch_pdl(k_chunk_sums, c->nchunk, 256, 0, c->s, v, (const int32_t*)w.chunk_lo,
                               (const int32_t*)w.chunk_hi, w.partial);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_replica_sums, (c->R + 127) / 128, 128, 0, c->s, c->R, (const int32_t*)w.chunk_rep,
                      c->nchunk, (const double*)w.partial, out, w.meta);
}

}  // namespace schnet
