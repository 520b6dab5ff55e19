// Atom-wise parts of SchNet: embedding, the interaction's in/out dense layers
// with the residual update, the per-atom readout, their backward pass, and the
// per-replica sums.  Rows are atoms; 64 atoms per CTA, fp32 throughout.
//
// Model reading (FlashSchNet paper-curation summary, How / Figure 2 caption:
// positions and embeddings pass through interaction blocks; readout per atom
// summed to the energy): h = x W_in; x += ssp(m Wo1 + bo1) Wo2 + bo2;
// eps = ssp(x R1 + c1) R2 + c2.  Backward (chain rule, by hand):
//   g^L = (ssp'(pr) (.) R2) R1^T;  u = ((g Wo2^T) (.) ssp'(q)) Wo1^T;
//   g^l = g^{l+1} + dh W_in^T.
#include "internal.h"

namespace schnet {

constexpr int AT = 64;           // atoms per CTA
constexpr int AW_THREADS = 256;

struct AWArgs {
    int N, T, L, layer;
    const int32_t* types;
    const float *emb, *Win, *Wo1, *Wo2, *WinT, *Wo1T, *Wo2T, *bo1, *bo2, *R1, *R1T, *c1, *R2, *c2;
    float *x, *h, *q, *m, *g, *dh, *pr, *eps;
    DevMeta* meta;
};

// C[64][NC] = A[64][KD] * B[KD][NC]; thread layout: 8 row groups x 32 column
// lanes; each thread owns rows rg*8..+7 and columns lane + 32 j.
template <int KD, int NC>
__device__ __forceinline__ void gemm64(const float* __restrict__ sA, const float* __restrict__ sB,
                                       float (&acc)[8][NC / 32])
{
    const int lane = threadIdx.x & 31, rg = threadIdx.x >> 5;
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int j = 0; j < NC / 32; ++j) acc[r][j] = 0.f;
#pragma unroll 4
    for (int k = 0; k < KD; ++k) {
        float b[NC / 32];
#pragma unroll
        for (int j = 0; j < NC / 32; ++j) b[j] = sB[k * NC + lane + 32 * j];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            float a = sA[(rg * 8 + r) * KD + k];
#pragma unroll
            for (int j = 0; j < NC / 32; ++j) acc[r][j] = fmaf(a, b[j], acc[r][j]);
        }
    }
}

__device__ __forceinline__ void load_mat(float* __restrict__ dst, const float* __restrict__ src, int n)
{
    const float4* s = reinterpret_cast<const float4*>(src);
    float4* d = reinterpret_cast<float4*>(dst);
    for (int i = threadIdx.x; i < n / 4; i += blockDim.x) d[i] = __ldg(s + i);
}

// load rows [i0, i0+64) of a [N][W] array into smem (zeros past N)
template <int W>
__device__ __forceinline__ void load_rows(float* __restrict__ dst, const float* __restrict__ src, int i0, int N)
{
    for (int idx = threadIdx.x; idx < AT * W / 4; idx += blockDim.x) {
        int r = idx / (W / 4);
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i0 + r < N) v = __ldg(reinterpret_cast<const float4*>(src + (size_t)(i0 + r) * W) + idx % (W / 4));
        reinterpret_cast<float4*>(dst)[idx] = v;
    }
}

#define AW_SMEM_FLOATS (FP * FP + 2 * AT * FP)

// x = emb[z]; h0 = x W_in[0]
__global__ void __launch_bounds__(AW_THREADS) k_aw_first(AWArgs a)
{
    extern __shared__ float sm[];
    float *sW = sm, *sX = sm + FP * FP;
    const int i0 = blockIdx.x * AT;
    const int lane = threadIdx.x & 31, rg = threadIdx.x >> 5;
    for (int idx = threadIdx.x; idx < AT * FP; idx += blockDim.x) {
        int r = idx / FP, f = idx % FP, i = i0 + r;
        float v = 0.f;
        if (i < a.N) {
            int z = a.types[i];
            if (z < 0 || z >= a.T) {
                if (f == 0) set_flag(a.meta, SCHNET_FLAG_BADTYPE);
                z = 0;
            }
            v = a.emb[z * FP + f];
            a.x[(size_t)i * FP + f] = v;
        }
        sX[idx] = v;
    }
    load_mat(sW, a.Win, FP * FP);
    __syncthreads();
    float acc[8][4];
    gemm64<FP, FP>(sX, sW, acc);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        int i = i0 + rg * 8 + r;
        if (i < a.N)
#pragma unroll
            for (int j = 0; j < 4; ++j) a.h[(size_t)i * FP + lane + 32 * j] = acc[r][j];
    }
}

// after the filter convolution of layer l:
//   q = m Wo1 + bo1; x += ssp(q) Wo2 + bo2; then h_{l+1} = x W_in or the readout.
__global__ void __launch_bounds__(AW_THREADS) k_aw_fwd(AWArgs a)
{
    extern __shared__ float sm[];
    float *sW = sm, *sX = sm + FP * FP, *sY = sX + AT * FP;
    const int l = a.layer, i0 = blockIdx.x * AT;
    const int lane = threadIdx.x & 31, rg = threadIdx.x >> 5;
    float* ql = a.q + (size_t)l * a.N * FP;
    load_rows<FP>(sX, a.m, i0, a.N);
    load_mat(sW, a.Wo1 + (size_t)l * FP * FP, FP * FP);
    __syncthreads();
    float acc[8][4];
    gemm64<FP, FP>(sX, sW, acc);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        int row = rg * 8 + r, i = i0 + row;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int f = lane + 32 * j;
            float qv = acc[r][j] + a.bo1[l * FP + f];
            if (i < a.N) ql[(size_t)i * FP + f] = qv;
            sY[row * FP + f] = ssp(qv);
        }
    }
    __syncthreads();
    load_mat(sW, a.Wo2 + (size_t)l * FP * FP, FP * FP);
    load_rows<FP>(sX, a.x, i0, a.N);
    __syncthreads();
    gemm64<FP, FP>(sY, sW, acc);
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        int row = rg * 8 + r, i = i0 + row;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int f = lane + 32 * j;
            float xv = sX[row * FP + f] + acc[r][j] + a.bo2[l * FP + f];
            sX[row * FP + f] = xv;
            if (i < a.N) a.x[(size_t)i * FP + f] = xv;
        }
    }
    if (l + 1 < a.L) {
        load_mat(sW, a.Win + (size_t)(l + 1) * FP * FP, FP * FP);
        __syncthreads();
        gemm64<FP, FP>(sX, sW, acc);
        float* hn = a.h + (size_t)(l + 1) * a.N * FP;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            int i = i0 + rg * 8 + r;
            if (i < a.N)
#pragma unroll
                for (int j = 0; j < 4; ++j) hn[(size_t)i * FP + lane + 32 * j] = acc[r][j];
        }
    } else {
        // readout: pr = x R1 + c1 (HP columns); eps = sum_k ssp(pr_k) R2_k + c2
        load_mat(sW, a.R1, FP * HP);
        __syncthreads();
        float acr[8][2];
        gemm64<FP, HP>(sX, sW, acr);
        const float c2 = a.c2[0];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            int i = i0 + rg * 8 + r;
            float part = 0.f;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                int k = lane + 32 * j;
                float p = acr[r][j] + a.c1[k];
                if (i < a.N) a.pr[(size_t)i * HP + k] = p;
                part += ssp(p) * a.R2[k];
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (lane == 0 && i < a.N) a.eps[i] = part + c2;
        }
    }
}

// u_{l} = ((g Wo2_l^T) (.) ssp'(q_l)) Wo1_l^T, with g held in sX; writes u into m.
__device__ __forceinline__ void bwd_to_u(const AWArgs& a, int l, int i0, float* sW, float* sX, float* sY)
{
    const int lane = threadIdx.x & 31, rg = threadIdx.x >> 5;
    const float* ql = a.q + (size_t)l * a.N * FP;
    float acc[8][4];
    __syncthreads();
    load_mat(sW, a.Wo2T + (size_t)l * FP * FP, FP * FP);
    __syncthreads();
    gemm64<FP, FP>(sX, sW, acc);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        int row = rg * 8 + r, i = i0 + row;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int f = lane + 32 * j;
            float qv = i < a.N ? ql[(size_t)i * FP + f] : 0.f;
            sY[row * FP + f] = acc[r][j] * sigmoidf(qv);
        }
    }
    __syncthreads();
    load_mat(sW, a.Wo1T + (size_t)l * FP * FP, FP * FP);
    __syncthreads();
    gemm64<FP, FP>(sY, sW, acc);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        int i = i0 + rg * 8 + r;
        if (i < a.N)
#pragma unroll
            for (int j = 0; j < 4; ++j) a.m[(size_t)i * FP + lane + 32 * j] = acc[r][j];
    }
}

// g^L from the readout, then u_{L-1}
__global__ void __launch_bounds__(AW_THREADS) k_aw_bwd_top(AWArgs a)
{
    extern __shared__ float sm[];
    float *sW = sm, *sX = sm + FP * FP, *sY = sX + AT * FP;
    const int i0 = blockIdx.x * AT;
    const int lane = threadIdx.x & 31, rg = threadIdx.x >> 5;
    // sY[64][HP] = ssp'(pr) (.) R2
    for (int idx = threadIdx.x; idx < AT * HP; idx += blockDim.x) {
        int r = idx / HP, k = idx % HP, i = i0 + r;
        float v = 0.f;
        if (i < a.N) v = sigmoidf(a.pr[(size_t)i * HP + k]) * a.R2[k];
        sY[idx] = v;
    }
    load_mat(sW, a.R1T, HP * FP);
    __syncthreads();
    float acc[8][4];
    gemm64<HP, FP>(sY, sW, acc);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        int row = rg * 8 + r, i = i0 + row;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int f = lane + 32 * j;
            sX[row * FP + f] = acc[r][j];
            if (i < a.N) a.g[(size_t)i * FP + f] = acc[r][j];
        }
    }
    bwd_to_u(a, a.L - 1, i0, sW, sX, sY);
}

// g^l = g^{l+1} + dh_l W_in_l^T, then u_{l-1} when l > 0
__global__ void __launch_bounds__(AW_THREADS) k_aw_bwd(AWArgs a)
{
    extern __shared__ float sm[];
    float *sW = sm, *sX = sm + FP * FP, *sY = sX + AT * FP;
    const int l = a.layer, i0 = blockIdx.x * AT;
    const int lane = threadIdx.x & 31, rg = threadIdx.x >> 5;
    load_rows<FP>(sY, a.dh, i0, a.N);
    load_mat(sW, a.WinT + (size_t)l * FP * FP, FP * FP);
    __syncthreads();
    float acc[8][4];
    gemm64<FP, FP>(sY, sW, acc);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        int row = rg * 8 + r, i = i0 + row;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int f = lane + 32 * j;
            float gv = acc[r][j] + (i < a.N ? a.g[(size_t)i * FP + f] : 0.f);
            sX[row * FP + f] = gv;
            if (i < a.N) a.g[(size_t)i * FP + f] = gv;
        }
    }
    if (l > 0) bwd_to_u(a, l - 1, i0, sW, sX, sY);
}

// ---------------------------------------------------------------------------
// per-replica sums (float64 accumulation, fixed order)
// ---------------------------------------------------------------------------
__global__ void k_chunk_sums(const float* __restrict__ v, const int32_t* __restrict__ lo,
                             const int32_t* __restrict__ hi, double* __restrict__ partial)
{
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
    int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= R) return;
    // chunks of replica r are contiguous; find them by scanning the (small) table
    double s = 0.0;
    for (int c = 0; c < nchunk; ++c)
        if (chunk_rep[c] == r) s += partial[c];
    out[r] = s;
    if (!isfinite(s)) set_flag(meta, SCHNET_FLAG_NONFINITE);
}

static AWArgs aw_args(schnet_ctx* c, const int32_t* types, int layer)
{
    Workspace& w = c->ws;
    AWArgs a;
    a.N = c->N; a.T = c->T; a.L = c->L; a.layer = layer;
    a.types = types;
    a.emb = w.emb; a.Win = w.Win; a.Wo1 = w.Wo1; a.Wo2 = w.Wo2;
    a.WinT = w.WinT; a.Wo1T = w.Wo1T; a.Wo2T = w.Wo2T;
    a.bo1 = w.bo1; a.bo2 = w.bo2; a.R1 = w.R1; a.R1T = w.R1T; a.c1 = w.c1; a.R2 = w.R2; a.c2 = w.c2;
    a.x = w.x; a.h = w.h; a.q = w.q; a.m = w.m; a.g = w.g; a.dh = w.dh; a.pr = w.pr; a.eps = w.eps;
    a.meta = w.meta;
    return a;
}

constexpr size_t AW_SMEM = sizeof(float) * AW_SMEM_FLOATS;

cudaError_t atomwise_init_attributes()
{
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k_aw_first, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)AW_SMEM))) return e;
    if ((e = cudaFuncSetAttribute(k_aw_fwd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)AW_SMEM))) return e;
    if ((e = cudaFuncSetAttribute(k_aw_bwd_top, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)AW_SMEM)))
        return e;
    return cudaFuncSetAttribute(k_aw_bwd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)AW_SMEM);
}

static int aw_blocks(schnet_ctx* c) { return (c->N + AT - 1) / AT; }

cudaError_t launch_aw_first(schnet_ctx* c, const int32_t* types)
{
    k_aw_first<<<aw_blocks(c), AW_THREADS, AW_SMEM, c->s>>>(aw_args(c, types, 0));
    c->launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_aw_fwd(schnet_ctx* c, int layer)
{
    k_aw_fwd<<<aw_blocks(c), AW_THREADS, AW_SMEM, c->s>>>(aw_args(c, nullptr, layer));
    c->launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_aw_bwd_top(schnet_ctx* c)
{
    k_aw_bwd_top<<<aw_blocks(c), AW_THREADS, AW_SMEM, c->s>>>(aw_args(c, nullptr, c->L - 1));
    c->launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_aw_bwd(schnet_ctx* c, int layer)
{
    k_aw_bwd<<<aw_blocks(c), AW_THREADS, AW_SMEM, c->s>>>(aw_args(c, nullptr, layer));
    c->launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_replica_sum(schnet_ctx* c, const float* v, double* out)
{
    Workspace& w = c->ws;
    k_chunk_sums<<<c->nchunk, 256, 0, c->s>>>(v, w.chunk_lo, w.chunk_hi, w.partial);
    k_replica_sums<<<(c->R + 127) / 128, 128, 0, c->s>>>(c->R, w.chunk_rep, c->nchunk, w.partial, out, w.meta);
    c->launches += 2;
    return cudaGetLastError();
}

}  // namespace schnet
