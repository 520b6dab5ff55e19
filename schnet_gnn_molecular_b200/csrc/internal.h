// Host-side context and launcher declarations shared by the library's .cu files.
#pragma once

#include <cmath>
#include <cstddef>
#include <cstdint>
#include <string>
#include <utility>
#include <vector>
#include <cuda_runtime.h>

#include "../../include/schnet.h"
#include "common.cuh"

namespace schnet {

constexpr int MAX_L = 8;
constexpr int GMAX_NONPERIODIC = 8;   // max cells per dimension of one replica's grid
constexpr int GMAX_PERIODIC = 256;
constexpr int SCAN_BLOCK = 1024;      // threads per scan block
constexpr int SCAN_ITEMS = 4;         // items per thread
constexpr int SCAN_TILE = SCAN_BLOCK * SCAN_ITEMS;
constexpr int REDUCE_CHUNK = 4096;    // atoms per partial sum of a per-replica reduction

// Cells are at least (r_c + skin) (1 + 2^-20) wide and atoms are binned in
// float64, so the binning's rounding (a few float64 ulps of the cell
// coordinate) can never put two atoms closer than r_c + skin two cells apart:
// the 27-cell stencil always sees every listed pair.
constexpr double CELL_MARGIN = 1.0 + 1.0 / 1048576.0;

// Cells of one grid dimension of length `ext` (host and device agree on it).
__host__ __device__ inline int cells_across(double ext, double rl, int gmax)
{
    const double q = ext / (rl * CELL_MARGIN);
    int g = q >= (double)gmax ? gmax : (int)floor(q);   // also catches +inf
    return g < 1 ? 1 : g;                                // and NaN, 0
}

// Cell-grid placement of one replica: cell coordinate u = (x - org) * inv.
struct GridGeom {
    double org[3];
    double inv[3];
};

// Per-layer packed tensor-core operand images (bytes) for the filter network.
constexpr size_t W1_IMG = (size_t)FP * KP * 2;   // one 16-bit term of W1^T (M=128 x K=64)
constexpr size_t W2_IMG = (size_t)FP * FP * 2;   // one 16-bit term of W2^T (M=128 x K=128)
constexpr size_t LAYER_IMG = 2 * W1_IMG + 2 * W2_IMG;  // hi + lo of both
// One atom-wise dense layer as an A operand: [128 rows][K = 128], hi term then lo term.
constexpr size_t AW_IMG = 2 * (size_t)FP * FP * 2;

struct Workspace {
    DevMeta* meta;
    // packed weights
    uint8_t* img;                 // [L][LAYER_IMG]
    float *s1, *s2, *b1;          // [L][FP] filter channel scales, first-layer bias
    float* b2;                    // [L][FP] second-layer bias (one 16-bit activation term: minus ln2 s2 sum_k W2^[k][f])
    float *emb;                   // [T][FP]
    float *emb_h0;                // [T][FP] emb W_in of interaction 0 (the first h of every atom of a type)
    uint8_t* aw_img;              // [6 L + 2][AW_IMG] atom-wise layers as tensor-core A operands
    float* aw_sc;                 // [6 L + 2][FP] their per-row scales
    float *bo1, *bo2;             // [L][FP]
    float *c1, *R2;               // [HP]
    float *c2;                    // [1]
    // atoms (pos4, ref4 and every activation below in slot order; frc4 in caller order)
    int32_t* atom_rep;            // [N]   replica of an atom (the same in both orders)
    int32_t* perm;                // [N]   caller index of the atom in each slot
    float4 *pos4, *ref4, *frc4;   // [N]
    // neighbour list
    int32_t *row_ptr, *rowcnt;    // [N+1]
    int32_t *hcnt, *rcnt;         // [N+1] per-row counts of the half list and its complement (scratch)
    int32_t *col, *coltmp, *rev, *erow;  // [cap]
    float* s_edge;                // [cap]
    int32_t *crow, *ccol, *cidx;  // [cap] edges with d < r_c, per CTA row range
    float* cdist;                 // [cap] their distances
    int32_t* ccount;              // [ncta]
    int32_t* part;                // [ncta+1]
    int32_t *crow_h, *ccol_h, *cidx_h;  // [cap] the half list: edges (i, j) that own their pair, d < r_c
    float* cdist_h;               // [cap] their distances
    int32_t* ccount_h;            // [ncta]    its per-CTA edge counts
    int32_t* part_h;              // [ncta+1]  and its own row partition
    int32_t *crow_r, *ccol_r;     // [cap] the complement: the other edges with d < r_c (dE/dh launches)
    float* cdist_r;               // [cap] their distances
    int32_t* ccount_r;            // [ncta]
    int32_t* part_r;              // [ncta+1]
    // cell list
    int32_t *cell_of, *cell_atoms;       // [N]  caller order
    int32_t* cell_slot;                  // [N]  cell of each slot
    int32_t *cell_cnt, *cell_start, *cell_fill;  // [ncell+1]
    int32_t* rep_off;             // [R+1] replica offsets
    int4* rgrid_dims;             // [R]   (gx, gy, gz, first cell)
    GridGeom* rgrid_geom;         // [R]   grid origin and inverse cell sizes (float64)
    long long* scan_tmp;          // [SCAN_TILE] tile sums
    // activations
    float *x, *h, *q, *m, *g, *pr, *eps, *ke;
    float *dh, *dh2;              // [N*FP] dE/dh: the half list's terms and the complement's
    // reductions
    double* partial;              // [nchunk]
    int32_t *chunk_rep, *chunk_lo, *chunk_hi;  // [nchunk]
    double *epot, *ekin;          // [R] scratch when caller passes NULL
    // host-step staging
    float *st_pos, *st_vel, *st_mass;  // [N*3], [N*3], [N]
    int32_t* st_types;                 // [N]
    double *st_epot, *st_ekin;         // [R]
};

struct GraphKey {
    const void *pos, *vel, *types, *mass, *epot, *ekin, *noise;
    float dt, gamma, temp;
    int n_rebuild;
    unsigned long long seed;
    bool operator==(const GraphKey& o) const
    {
        return pos == o.pos && vel == o.vel && types == o.types && mass == o.mass && epot == o.epot &&
               ekin == o.ekin && noise == o.noise && dt == o.dt && gamma == o.gamma && temp == o.temp &&
               n_rebuild == o.n_rebuild && seed == o.seed;
    }
};

// Launch on `s` with programmatic stream serialization: the kernel's CTAs may be
// scheduled while the previous kernel on the stream is still finishing, run
// their prologue on data no kernel of the step writes, and wait in pdl_wait for
// its results.  Every kernel launched this way calls pdl_wait before reading
// anything an earlier kernel of the step wrote and before writing anything an
// earlier kernel reads.  The neighbour build's kernels are launched without it,
// so they have completed before the next kernel starts.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t s,
                              Args... args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace schnet

struct schnet_ctx {
    schnet_config cfg;
    std::vector<int32_t> rep_off;   // host copy [R+1]
    int N, R, T, F, K, L, H;
    int weight_fmt;                 // 0 fp16 operands, 1 bf16 operands
    int n_wterms;                   // 2 (fp32 storage: hi+lo) or 1
    int n_xterms;                   // filter activations: 2 (hi+lo) or 1 (16-bit, the fast mode)
    int64_t cap;
    int nsm, ncta;                  // SMs; CTAs of the tensor-core kernels
    int ncell;                      // total cells reserved
    int nchunk;                     // per-replica reduction chunks
    int gdim[3];                    // periodic grid dims
    double rl2;                     // (cutoff + skin)^2 in float64
    float mu0, dmu;                 // Gaussian centres mu_k = mu0 + k dmu
    schnet::Box box;
    cudaStream_t user_stream;
    cudaStream_t s;                 // internal stream
    cudaEvent_t ev_in, ev_out;
    schnet::Workspace ws;
    bool have_list = false;
    bool forces_valid = false;
    // MD phase: steps taken since the last neighbour build
    int since_build = 0;
    // graph cache: 0 = build + n_rebuild steps, 1 = build + one step, 2 = one step
    struct GraphSlot {
        bool ok = false;
        schnet::GraphKey key{};
        cudaGraphExec_t exec = nullptr;
        int64_t kernels = 0;
    } graphs[3];
    int64_t launches = 0;
    // profiling (schnet_profile_steps): event pairs per kernel class
    bool prof = false;
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> prof_pairs[SCHNET_KERNEL_NCLASS];
    std::string err;
};

namespace schnet {

// launchers (each enqueues on ctx->s and counts its kernels in ctx->launches)
cudaError_t launch_pack_positions(schnet_ctx* c, const float* d_pos);
cudaError_t launch_build_neighbors(schnet_ctx* c, const float* d_pos);
cudaError_t launch_caller_order_list(schnet_ctx* c, const int32_t** row_ptr, const int32_t** col,
                                     const int32_t** rev);
cudaError_t launch_scatter_atoms(schnet_ctx* c, const float* v, float* out);
cudaError_t launch_test_timeout(schnet_ctx* c, uint32_t max_polls, int complete);
cudaError_t launch_energy_forces(schnet_ctx* c, const int32_t* d_types, double* d_energy, float* d_forces,
                                 bool need_forces, bool sum_energy = true);
cudaError_t launch_baoa(schnet_ctx* c, float* d_pos, float* d_vel, const float* d_mass, float dt, float gamma,
                        float temp, unsigned long long seed, const float* d_noise, bool check_skin);
cudaError_t launch_b_kick(schnet_ctx* c, float* d_vel, const float* d_mass, float dt, double* d_ekin,
                          bool sum_ke = true);
cudaError_t launch_set_step(schnet_ctx* c, unsigned long long step);
cudaError_t launch_forces(schnet_ctx* c, float* d_forces);
cudaError_t launch_replica_sum(schnet_ctx* c, const float* v, double* out);
cudaError_t launch_embed(schnet_ctx* c, const int32_t* types);
cudaError_t launch_aw_fwd(schnet_ctx* c, int layer);
cudaError_t launch_aw_bwd_top(schnet_ctx* c);
cudaError_t launch_aw_bwd(schnet_ctx* c, int layer);
cudaError_t launch_compact(schnet_ctx* c, bool with_half);
cudaError_t launch_cfconv_fwd(schnet_ctx* c, int layer);
cudaError_t launch_cfconv_dh(schnet_ctx* c, int layer);
cudaError_t launch_cfconv_pair(schnet_ctx* c, int layer, int accumulate_s, bool with_dh);
cudaError_t cfconv_init_attributes();
cudaError_t atomwise_init_attributes();

}  // namespace schnet
