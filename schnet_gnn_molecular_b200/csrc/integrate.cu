// Forces from the per-edge scalars of the backward pass, and the Langevin /
// velocity-Verlet update of many replicas at once.
//
// Forces: the backward kernels leave, on the owning edge e = (i, j) (owns_pair), of
// every pair within the cutoff, its derivative dE/dd_ij summed over the
// interactions (the half list visits each pair once); and
// F_i = sum_{e in row i} dE/dd_ij (r_j - r_i) / d_ij, with the value read from
// e or from its transpose rev(e) -- a per-row segment sum over the CSR, no
// atomics (FlashSchNet paper-curation summary, How: contention-free
// accumulation forward and backward).
// Rows are slots (atoms in cell order); perm maps a slot to the caller's
// index, under which forces are stored for the integrator and the caller.
// Integrator (the pages name Langevin / velocity-Verlet dynamics but give no
// scheme): BAOAB of Leimkuhler & Matthews; gamma = 0 is velocity Verlet.
// Noise: Philox4x32-10 (Salmon et al., SC'11) keyed by the seed, counter
// (atom, step), Box-Muller in float64.
#include "internal.h"

namespace schnet {

constexpr float ACC = 4.184e-4f;          // (kcal/mol/A)/amu -> A/fs^2
constexpr double KB = 0.0019872041;       // kcal/mol/K

__global__ void k_forces(int n, const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                         const int32_t* __restrict__ rev, const float* __restrict__ s_edge,
                         const float4* __restrict__ pos4, const int32_t* __restrict__ perm, const Box box,
                         float rc, long long cap, DevMeta* meta, float4* __restrict__ frc4,
                         float* __restrict__ out3)
{
    pdl_trigger();
    pdl_wait();
    if (meta->n_edges > cap) return;
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int i = warp; i < n; i += nwarps) {
        const float4 pi = pos4[i];
        float fx = 0.f, fy = 0.f, fz = 0.f;
        const int a = row_ptr[i], b = row_ptr[i + 1];
        for (int e = a + lane; e < b; e += 32) {
            const int j = col[e];
            float3 v;
            const float d = edge_distance(pi, pos4[j], box, v);
            if (d < rc && d > 0.f) {
                // the pair's derivative sits on its owning edge
                const int re = rev[e];
                const float D = owns_pair(i, j) ? s_edge[e] : (re >= 0 ? s_edge[re] : 0.f);
                float k = D / d;
                fx = fmaf(k, v.x, fx);
                fy = fmaf(k, v.y, fy);
                fz = fmaf(k, v.z, fz);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            fx += __shfl_xor_sync(0xffffffffu, fx, o);
            fy += __shfl_xor_sync(0xffffffffu, fy, o);
            fz += __shfl_xor_sync(0xffffffffu, fz, o);
        }
        if (lane == 0) {
            const int ic = perm[i];
            frc4[ic] = make_float4(fx, fy, fz, 0.f);
            if (out3) {
                out3[3 * ic] = fx;
                out3[3 * ic + 1] = fy;
                out3[3 * ic + 2] = fz;
            }
            if (!(isfinite(fx) && isfinite(fy) && isfinite(fz))) set_flag(meta, SCHNET_FLAG_NONFINITE);
        }
    }
}

cudaError_t launch_forces(schnet_ctx* c, float* d_forces)
{
    Workspace& w = c->ws;
    int blocks = (c->N + 7) / 8;   // 8 warps per block, one row per warp
    if (blocks > c->nsm * 16) blocks = c->nsm * 16;
    c->launches += 1;
    return launch_pdl(k_forces, blocks, 256, 0, c->s, c->N, (const int32_t*)w.row_ptr, (const int32_t*)w.col,
                      (const int32_t*)w.rev, (const float*)w.s_edge, (const float4*)w.pos4, (const int32_t*)w.perm,
                      c->box, c->cfg.cutoff, (long long)c->cap, w.meta, w.frc4, d_forces);
}

// --- Philox4x32-10 -----------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 ctr, uint2 key)
{
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u, W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            key.x += W0;
            key.y += W1;
        }
        uint32_t hi0 = __umulhi(M0, ctr.x), lo0 = M0 * ctr.x;
        uint32_t hi1 = __umulhi(M1, ctr.z), lo1 = M1 * ctr.z;
        ctr = make_uint4(hi1 ^ ctr.y ^ key.x, lo1, hi0 ^ ctr.w ^ key.y, lo0);
    }
    return ctr;
}

__device__ __forceinline__ float3 normals3(unsigned long long seed, unsigned long long step, int i)
{
    uint4 o = philox4x32_10(make_uint4((uint32_t)i, (uint32_t)step, (uint32_t)(step >> 32), 0u),
                            make_uint2((uint32_t)seed, (uint32_t)(seed >> 32)));
    const double s = 2.3283064365386963e-10;   // 2^-32
    double u0 = ((double)o.x + 1.0) * s, u1 = ((double)o.y + 1.0) * s;
    double u2 = ((double)o.z + 1.0) * s, u3 = ((double)o.w + 1.0) * s;
    double r0 = sqrt(-2.0 * log(u0)), r1 = sqrt(-2.0 * log(u2));
    double s1, c1, s3, c3;
    sincospi(2.0 * u1, &s1, &c1);
    sincospi(2.0 * u3, &s3, &c3);
    return make_float3((float)(r0 * c1), (float)(r0 * s1), (float)(r1 * c3));
}

// B (half kick with the current forces), A, O, A.  One thread per slot k: the
// atom's caller index i addresses the caller's arrays and the noise counter,
// k the slot-order positions of the force evaluation and the skin reference.
__global__ void k_baoa(int n, const int32_t* __restrict__ perm, float* __restrict__ pos, float* __restrict__ vel,
                       const float* __restrict__ mass, const float4* __restrict__ frc4, float4* __restrict__ pos4,
                       const float4* __restrict__ ref4, float dt, float c1, float kT_acc, int langevin,
                       unsigned long long seed, const float* __restrict__ noise, int check_skin, float half_skin2,
                       DevMeta* meta)
{
    pdl_trigger();
    pdl_wait();
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= n) return;
    const int i = perm[k];
    const float inv_m = 1.0f / mass[i];
    const float4 F = frc4[i];
    const float hk = 0.5f * dt * ACC * inv_m;
    float v[3] = {vel[3 * i], vel[3 * i + 1], vel[3 * i + 2]};
    float r[3] = {pos[3 * i], pos[3 * i + 1], pos[3 * i + 2]};
    const float f[3] = {F.x, F.y, F.z};
    float3 xi = make_float3(0.f, 0.f, 0.f);
    if (langevin) {
        if (noise) xi = make_float3(noise[3 * i], noise[3 * i + 1], noise[3 * i + 2]);
        else xi = normals3(seed, meta->step, i);
    }
    const float sv = sqrtf((1.0f - c1 * c1) * kT_acc * inv_m);
    const float x3[3] = {xi.x, xi.y, xi.z};
#pragma unroll
    for (int d = 0; d < 3; ++d) {
        float vv = fmaf(hk, f[d], v[d]);
        float rr = fmaf(0.5f * dt, vv, r[d]);
        if (langevin) vv = fmaf(c1, vv, sv * x3[d]);
        rr = fmaf(0.5f * dt, vv, rr);
        v[d] = vv;
        r[d] = rr;
    }
#pragma unroll
    for (int d = 0; d < 3; ++d) {
        vel[3 * i + d] = v[d];
        pos[3 * i + d] = r[d];
    }
    pos4[k] = make_float4(r[0], r[1], r[2], 0.f);
    if (!(isfinite(r[0]) && isfinite(r[1]) && isfinite(r[2]))) set_flag(meta, SCHNET_FLAG_NONFINITE);
    if (check_skin) {
        float4 q = ref4[k];
        float dx = r[0] - q.x, dy = r[1] - q.y, dz = r[2] - q.z;
        if (dx * dx + dy * dy + dz * dz > half_skin2) set_flag(meta, SCHNET_FLAG_SKIN);
    }
}

cudaError_t launch_baoa(schnet_ctx* c, float* d_pos, float* d_vel, const float* d_mass, float dt, float gamma,
                        float temp, unsigned long long seed, const float* d_noise, bool check_skin)
{
    Workspace& w = c->ws;
    double c1 = exp(-(double)gamma * 1e-3 * (double)dt);
    double kT_acc = KB * (double)temp * (double)ACC;
    float hs = 0.5f * c->cfg.skin;
    c->launches += 1;
    return launch_pdl(k_baoa, (c->N + 255) / 256, 256, 0, c->s, c->N, (const int32_t*)w.perm, d_pos, d_vel, d_mass,
                      (const float4*)w.frc4, w.pos4, (const float4*)w.ref4, dt, (float)c1, (float)kT_acc,
                      gamma != 0.f ? 1 : 0, (unsigned long long)seed, d_noise, check_skin ? 1 : 0, hs * hs, w.meta);
}

// closing half kick; per-atom kinetic energy (kcal/mol) into tmp; step += 1
__global__ void k_b_kick(int n, float* __restrict__ vel, const float* __restrict__ mass,
                         const float4* __restrict__ frc4, float dt, float* __restrict__ ke, DevMeta* meta)
{
    pdl_trigger();
    pdl_wait();
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i == 0) meta->step += 1ull;
    if (i >= n) return;
    const float m = mass[i];
    const float hk = 0.5f * dt * ACC / m;
    const float4 F = frc4[i];
    float vx = fmaf(hk, F.x, vel[3 * i]);
    float vy = fmaf(hk, F.y, vel[3 * i + 1]);
    float vz = fmaf(hk, F.z, vel[3 * i + 2]);
    vel[3 * i] = vx;
    vel[3 * i + 1] = vy;
    vel[3 * i + 2] = vz;
    ke[i] = 0.5f * m * (vx * vx + vy * vy + vz * vz) * (1.0f / ACC);
}

cudaError_t launch_replica_sum(schnet_ctx* c, const float* v, double* out);

cudaError_t launch_b_kick(schnet_ctx* c, float* d_vel, const float* d_mass, float dt, double* d_ekin, bool sum_ke)
{
    Workspace& w = c->ws;
    c->launches += 1;
    cudaError_t e = launch_pdl(k_b_kick, (c->N + 255) / 256, 256, 0, c->s, c->N, d_vel, d_mass, (const float4*)w.frc4,
                               dt, w.ke, w.meta);
    if (e != cudaSuccess || !sum_ke) return e;
    return launch_replica_sum(c, w.ke, d_ekin ? d_ekin : w.ekin);
}

__global__ void k_set_step(DevMeta* meta, unsigned long long step) { meta->step = step; }

cudaError_t launch_set_step(schnet_ctx* c, unsigned long long step)
{
    k_set_step<<<1, 1, 0, c->s>>>(c->ws.meta, step);
    c->launches += 1;
    return cudaGetLastError();
}

}  // namespace schnet
