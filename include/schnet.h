/*
 * schnet.h -- C ABI of the B200 SchNet CFConv energy / force / integrate library.
 *
 * What is computed (sources are the pages' titles and sections):
 *   "FlashSchNet: Fast and Accurate Coarse-Grained Neural Network Molecular
 *   Dynamics" (paper-curation summary), section How, and the same work's
 *   abstract (OpenAlex record): a SchNet-style GNN potential over coarse-grained
 *   beads; per edge the pairwise distance, a Gaussian radial-basis expansion
 *   and a cosine envelope (flash radial basis), the filter network, cutoff
 *   masking, neighbour gather, filter multiplication and a CSR segment
 *   reduction per atom (flash message passing / flash aggregation, forward
 *   and backward); forces from the backward pass; many independent replicas
 *   advanced together (section Achievement 1).  "Ab Initio Accuracy Beyond
 *   the Cutoff" (Tessera), abstract: a conservative neighbour skin keeps the
 *   graph fixed between rebuilds so each rebuild interval replays as one CUDA
 *   Graph.
 * Model (plain SchNet reading, all dense weights row-major [in][out]):
 *   x0_i = emb[z_i];  per interaction l: h = x W_in_l,
 *   W(d) = f_c(d) (ssp(e(d) W1_l + b1_l) W2_l + b2_l),
 *   e_k(d) = exp(-(d - mu_k)^2 / (2 sigma^2)), mu_k evenly spaced on
 *   [rbf_min, rbf_max] (both included), f_c(d) = (cos(pi d / r_c) + 1) / 2
 *   for d < r_c else 0, ssp(x) = ln(1 + e^x) - ln 2;
 *   m_i = sum_{j: d_ij < r_c} h_j (.) W(d_ij);  x += ssp(m Wo1_l + bo1_l) Wo2_l + bo2_l;
 *   eps_i = ssp(x R1 + c1) R2 + c2 (hidden width F/2);  E_r = sum_{i in r} eps_i;
 *   F_i = -dE/dr_i.
 * Units: Angstrom, fs, amu, kcal/mol, K.
 *
 * Conventions for every call:
 *   - Device pointers ("d_") point to memory of the device current at
 *     schnet_create; host pointers ("h_") to ordinary or pinned host memory.
 *   - Work is enqueued on the stream given to schnet_create and is ordered
 *     after prior work on it; calls return before the device finishes unless
 *     stated otherwise.  The library uses an internal stream joined to the
 *     caller's stream with events.
 *   - The caller owns every device buffer, including the workspace; the
 *     library owns only the schnet_ctx host object and its CUDA stream,
 *     events and graphs.  The library never calls cudaMalloc.
 *   - Argument errors are reported at once through the return value; errors
 *     detected on the device are sticky bits of a device status word (see
 *     SCHNET_FLAG_*), read back by schnet_get_status and at the end of
 *     schnet_step.  No call traps the GPU.
 */
#ifndef SCHNET_B200_H
#define SCHNET_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SCHNET_API __attribute__((visibility("default")))
#else
#define SCHNET_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SCHNET_OK = 0,
    SCHNET_ERR_INVALID_ARG = 1,  /* bad pointer, size or configuration            */
    SCHNET_ERR_CUDA = 2,         /* a CUDA runtime call failed (see last_error)    */
    SCHNET_ERR_CAPACITY = 3,     /* edge list overflowed edge_capacity             */
    SCHNET_ERR_SKIN = 4,         /* an atom moved more than skin/2 since the build */
    SCHNET_ERR_NONFINITE = 5,    /* NaN/Inf in energies, forces or positions       */
    SCHNET_ERR_BADTYPE = 6,      /* a bead type outside [0, n_types)               */
    SCHNET_ERR_STATE = 7,        /* call order (e.g. no neighbour list yet)        */
    SCHNET_ERR_TIMEOUT = 8,      /* a bounded device-side wait gave up             */
    SCHNET_ERR_UNSUPPORTED = 9   /* configuration outside the supported envelope   */
} schnet_status;

/* Bits of the device status word. */
#define SCHNET_FLAG_CAPACITY  0x1u
#define SCHNET_FLAG_SKIN      0x2u
#define SCHNET_FLAG_NONFINITE 0x4u
#define SCHNET_FLAG_BADTYPE   0x8u
#define SCHNET_FLAG_TIMEOUT   0x10u

/* Filter-network weight storage (flag for channel-wise 16-bit weights,
 * FlashSchNet summary, How: "channel-wise 16-bit quantization").  Each
 * output channel o of W1 and W2 is scaled by s_o = max_i |W[i][o]|
 * (fp32 scales, fp32 accumulation).
 *   FP32: the scaled weights are carried as an fp16 hi + lo pair (about 22
 *         significant bits) and activations likewise: fp32-level accuracy on
 *         the 16-bit tensor-core path.
 *   FP16 / BF16: the scaled weights are rounded once to the 16-bit type
 *         (what is stored), activations still carried as hi + lo pairs.
 *   FP16_FAST: fp16 weights as FP16, and the filter network's activations
 *         (Gaussians, their distance derivatives, the softplus outputs and
 *         their tangents) rounded once to fp16 as well: one tensor-core
 *         product per K-step instead of two (FP16) or three (FP32).  The
 *         atom-wise layers and all accumulations stay fp32.  A speed mode,
 *         held to the 16-bit tolerance (forces within 2e-3 of fp32). */
typedef enum {
    SCHNET_WEIGHTS_FP32 = 0,
    SCHNET_WEIGHTS_FP16 = 1,
    SCHNET_WEIGHTS_BF16 = 2,
    SCHNET_WEIGHTS_FP16_FAST = 3
} schnet_weight_dtype;

typedef struct {
    int32_t n_types;          /* T  >= 1                                       */
    int32_t n_features;       /* F, even, 2..128                               */
    int32_t n_rbf;            /* K, 1..64                                      */
    int32_t n_interactions;   /* L, 1..8                                       */
    float rbf_min, rbf_max;   /* Gaussian centres span [rbf_min, rbf_max], A   */
    float rbf_sigma;          /* Gaussian width sigma, A                       */
    float cutoff;             /* r_c, A                                        */
    float skin;               /* neighbour-list skin, A (list radius r_c+skin) */
    int32_t periodic;         /* 1: orthorhombic box, minimum image            */
    float box[3];             /* box lengths, A (periodic only; >= 2 (r_c+skin)) */
    int32_t n_atoms;          /* N, total beads over all replicas              */
    int32_t n_replicas;       /* R >= 1                                        */
    const int32_t *replica_offsets; /* host [R+1], 0 = o_0 <= ... <= o_R = N; replica r
                                       owns atoms [o_r, o_{r+1}); read during create only */
    int64_t edge_capacity;    /* listed directed edges to reserve; 0: derived  */
    int32_t weight_dtype;     /* schnet_weight_dtype                          */
} schnet_config;

/* Host float32 weights, row-major [in][out], read during schnet_create only.
 * Shapes: emb [T][F]; W_in, W2, Wo1, Wo2 [L][F][F]; W1 [L][K][F];
 * b1, b2, bo1, bo2 [L][F]; R1 [F][F/2]; c1, R2 [F/2]; c2 scalar. */
typedef struct {
    const float *emb, *W_in, *W1, *b1, *W2, *b2, *Wo1, *bo1, *Wo2, *bo2, *R1, *c1, *R2;
    float c2;
} schnet_weights;

typedef struct schnet_ctx schnet_ctx;

/* Device workspace bytes needed for cfg (256-byte aligned base required).
 * Holds the neighbour list (col, rev, edge rows: edge_capacity entries each),
 * saved activations (L x N x 128 floats twice), packed weights and the status
 * word.  Errors: INVALID_ARG, UNSUPPORTED. */
SCHNET_API schnet_status schnet_workspace_bytes(const schnet_config *cfg, size_t *bytes);

/* Create a context on the current device.  cuda_stream: a cudaStream_t (NULL =
 * legacy default stream).  d_workspace: caller-owned device buffer of at
 * least schnet_workspace_bytes(cfg) bytes, kept alive until schnet_destroy.
 * Packs (and for 16-bit storage quantizes) the weights on the host in float64
 * and uploads them into the workspace; blocks until the upload is done.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.  On error *out is NULL. */
SCHNET_API schnet_status schnet_create(const schnet_config *cfg, const schnet_weights *w, void *cuda_stream,
                            void *d_workspace, size_t ws_bytes, schnet_ctx **out);

/* Build the neighbour list at positions d_pos (device float32 [N][3]):
 * all ordered pairs (i, j), i != j, of one replica with d_ij^2 < (r_c + skin)^2,
 * the test done in float64 from the float32 coordinates with each operation
 * rounded separately (dx = x_j - x_i, periodic dx -= L rint(dx / L),
 * d2 = (dx dx + dy dy) + dz dz).  Result: a destination-sorted CSR (row i lists
 * j ascending) plus rev[e] = index of the reverse edge (j, i), i.e. the
 * transposed list; a cell list (cells >= r_c + skin) limits the candidates.
 * The list is kept on the device with its edge count; positions are
 * snapshotted for the skin check.  Until the next build the context holds
 * atoms internally in cell order (cells grouped by replica, ascending atom
 * index inside a cell) so that atoms close in space are close in memory;
 * every value it returns (forces, energies, the taps below) is in the
 * caller's atom order.  Overflow sets SCHNET_FLAG_CAPACITY and leaves the
 * list unusable until a build fits.  Errors: INVALID_ARG, CUDA. */
SCHNET_API schnet_status schnet_build_neighbors(schnet_ctx *ctx, const float *d_pos);

/* Energy per replica and forces at d_pos using the current list.
 * d_types: device int32 [N]; d_energy: device float64 [R] (kcal/mol);
 * d_forces: device float32 [N][3] (kcal/mol/A), may be NULL for energy only (then no backward
 * pass runs).
 * Sets SCHNET_FLAG_SKIN if an atom moved more than skin/2 since the build,
 * SCHNET_FLAG_BADTYPE for a type outside [0, T) (treated as type 0).
 * Errors: INVALID_ARG, STATE (no list built), CUDA. */
SCHNET_API schnet_status schnet_energy_forces(schnet_ctx *ctx, const float *d_pos, const int32_t *d_types,
                                   double *d_energy, float *d_forces);

typedef struct {
    float dt_fs;          /* timestep, fs                                      */
    float gamma_per_ps;   /* Langevin friction, 1/ps; 0 = velocity Verlet      */
    float temperature_K;  /* bath temperature, K (ignored when gamma = 0)      */
    int32_t n_rebuild;    /* steps between neighbour rebuilds (>= 1)           */
    uint64_t seed;        /* Philox4x32-10 key                                  */
    uint64_t step0;       /* index of the first step (noise counter)           */
    const float *d_noise; /* optional device [N][3] normals used at every step
                             instead of Philox (testing); NULL = Philox         */
    int32_t resume;       /* 1: positions/velocities continue the previous call
                             on this context unchanged, reuse its forces       */
    int32_t use_graph;    /* 1: replay each rebuild interval as one CUDA Graph */
} schnet_step_params;

/* Advance n_steps BAOAB Langevin steps (Leimkuhler-Matthews order
 * B A O A [forces] B; gamma = 0 is velocity Verlet).  Noise: for atom i at
 * step s, Philox4x32-10 with key (seed lo, seed hi) and counter
 * (i, s lo, s hi, 0); outputs x_a -> u_a = (x_a + 1) / 2^32, Box-Muller gives
 * xi = (r0 cos 2 pi u1, r0 sin 2 pi u1, r1 cos 2 pi u3), r = sqrt(-2 ln u).
 * The list is rebuilt at the start of every interval of n_rebuild steps.
 * d_pos, d_vel: device float32 [N][3] updated in place (A, A/fs);
 * d_types int32 [N]; d_mass float32 [N] (amu); d_epot, d_ekin: device float64
 * [R] for the last step (may be NULL; the sums are formed at the last step
 * only).  Blocks at the end to read the status word once: returns
 * SKIN/CAPACITY/NONFINITE/BADTYPE/TIMEOUT if the corresponding flag was raised
 * during the call (flags then cleared).
 * Errors: INVALID_ARG, CUDA, or a flag status as above. */
SCHNET_API schnet_status schnet_step(schnet_ctx *ctx, float *d_pos, float *d_vel, const int32_t *d_types,
                          const float *d_mass, int64_t n_steps, const schnet_step_params *p,
                          double *d_epot, double *d_ekin);

/* Same as schnet_step on HOST buffers: copies h_pos, h_vel, h_types, h_mass
 * into workspace staging buffers, runs the steps, copies h_pos, h_vel and
 * (if non-NULL) h_epot, h_ekin back, and synchronizes. */
SCHNET_API schnet_status schnet_step_host(schnet_ctx *ctx, float *h_pos, float *h_vel, const int32_t *h_types,
                               const float *h_mass, int64_t n_steps, const schnet_step_params *p,
                               double *h_epot, double *h_ekin);

/* Synchronize the context's stream and return (then clear) the status word. */
SCHNET_API schnet_status schnet_get_status(schnet_ctx *ctx, uint32_t *flags);

/* Text of the last host-side error on this context ("" if none). */
SCHNET_API const char *schnet_last_error(const schnet_ctx *ctx);

/* Release the context (synchronizes; the workspace stays the caller's). */
SCHNET_API schnet_status schnet_destroy(schnet_ctx *ctx);

/* Test tap: synchronize and copy the current list, in the caller's atom order
 * (row i lists j ascending, as schnet_build_neighbors defines it), to host
 * arrays: h_row_ptr int32 [N+1], h_col, h_rev int32 [cap]; *n_edges = edge
 * count.  Any pointer may be NULL.  The reordering uses scratch that the next
 * evaluation rewrites anyway.  Errors: STATE (no list), CAPACITY if cap is
 * smaller than the list. */
SCHNET_API schnet_status schnet_get_neighbors(schnet_ctx *ctx, int32_t *h_row_ptr, int32_t *h_col, int32_t *h_rev,
                                   int64_t *n_edges, int64_t cap);

/* Test tap: per-atom energies eps_i of the last evaluation, device float32 [N],
 * caller's atom order.  Errors: INVALID_ARG, STATE (no list), CUDA. */
SCHNET_API schnet_status schnet_get_atom_energies(schnet_ctx *ctx, float *d_eps);

/* Test tap: d_y[i] = 2^d_x[i] (device float32 arrays of n elements, d_x[i] <= 0;
 * arguments below -30 are taken as -30) by the FMA-pipe exponential that part of
 * the forward filter's softplus uses, enqueued on cuda_stream (a cudaStream_t,
 * NULL = legacy default stream).  Errors: INVALID_ARG, CUDA. */
SCHNET_API schnet_status schnet_test_exp2(const float *d_x, float *d_y, int64_t n, void *cuda_stream);

/* Test tap: the give-up path of the library's device-side waits, on its own.  One
 * CTA holds tensor memory and waits on an mbarrier for at most max_polls polls;
 * with complete = 0 nothing completes the barrier, so the wait gives up, raises
 * SCHNET_FLAG_TIMEOUT in the context's status word, releases the tensor memory and
 * returns (complete = 1: the barrier completes at once, no flag).  Read the flag
 * with schnet_get_status; the context stays usable.  Errors: INVALID_ARG, CUDA. */
SCHNET_API schnet_status schnet_test_timeout(schnet_ctx *ctx, uint32_t max_polls, int32_t complete);

/* Kernel classes reported by schnet_profile_steps. */
enum {
    SCHNET_KERNEL_CFCONV_FWD = 0,  /* fused radial basis + filter MLP + message passing, forward */
    SCHNET_KERNEL_CFCONV_BWD = 1,  /* pair derivatives dE/dd (and the half list's dE/dh terms)  */
    SCHNET_KERNEL_ATOMWISE = 2,    /* embedding, atom-wise dense layers, readout (fwd + bwd)   */
    SCHNET_KERNEL_NEIGHBORS = 3,   /* one whole neighbour build (cell list, CSR, rev)          */
    SCHNET_KERNEL_FORCES = 4,      /* force assembly from the per-edge scalars                 */
    SCHNET_KERNEL_INTEGRATE = 5,   /* B-A-O-A and closing B kicks                              */
    SCHNET_KERNEL_REDUCE = 6,      /* per-replica energy sums                                  */
    SCHNET_KERNEL_MASK = 7,        /* per-step cutoff masking into the full, half, complement lists */
    SCHNET_KERNEL_CFCONV_DH = 8,   /* dE/dh over the complementary list (forward kernel, dE/dm) */
    SCHNET_KERNEL_NCLASS = 9
};

/* Profiling pass: continue the trajectory for n_steps steps exactly as
 * schnet_step would (resume semantics), but launched eagerly with a CUDA event
 * pair on the library's own stream around every kernel (a whole build counts
 * as one).  Synchronizes, then writes per class the summed device time in
 * milliseconds (ms_total[SCHNET_KERNEL_NCLASS]) and the number of timed
 * launches (launches[SCHNET_KERNEL_NCLASS]).  Errors as schnet_step. */
SCHNET_API schnet_status schnet_profile_steps(schnet_ctx *ctx, float *d_pos, float *d_vel, const int32_t *d_types,
                                              const float *d_mass, int64_t n_steps, const schnet_step_params *p,
                                              double *ms_total, int64_t *launches);

/* Neighbour list without any device allocation and without a context.
 * The pages have no counterpart to this entry point: it exists for callers
 * that cannot allocate device memory where they call the library (a host
 * program that only hands over buffers it already owns, or a runtime that
 * forbids cudaMalloc while it runs).  It builds the same list as
 * schnet_build_neighbors (same pair test, rows sorted, rev = transpose map),
 * with all scratch in one fixed array of about 3.6 MB that every device
 * loading this library keeps until the process exits.
 *   d_pos: device float32 [n_atoms][3]; d_replica_offsets: device int32
 *   [n_replicas+1] (0 .. n_atoms, non-decreasing); box: host float[3]
 *   (periodic only).  Outputs (caller-owned device buffers): d_row_ptr int32
 *   [n_atoms+1], d_col and d_rev int32 [edge_capacity], d_n_edges int64 [1]
 *   = edges found; if that exceeds edge_capacity, col and rev are not
 *   written and the caller should retry with more room.  d_flags (device
 *   uint32 [1], may be NULL) receives the SCHNET_FLAG_* bits of this call:
 *   SCHNET_FLAG_NONFINITE when a position is NaN or infinite (the list is then
 *   built with those atoms binned into an arbitrary cell, so it may miss
 *   pairs and should not be used), SCHNET_FLAG_CAPACITY when the list did not
 *   fit.  Both outputs are written on the stream; read them after it syncs.
 * Limits: n_atoms <= 65536, n_replicas <= 1024, cells <= 131072 (open
 * boundaries use 512 cells per replica, so n_replicas <= 256 there),
 * edge_capacity < 2^31; larger inputs return SCHNET_ERR_UNSUPPORTED, bad
 * pointers or sizes SCHNET_ERR_INVALID_ARG.  Asynchronous on cuda_stream.
 * A CUDA error already pending on the calling thread when the call starts is
 * left in place and reported as SCHNET_ERR_CUDA before anything is enqueued.
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.
 * Every call reuses the same array and zeroes what must start at zero, so
 * calls that overlap on the GPU (other streams or other host threads)
 * race and must be serialized by the caller.  No call allocates memory. */
SCHNET_API schnet_status schnet_build_neighbors_noalloc(const float *d_pos, int32_t n_atoms, int32_t n_replicas,
                                                        const int32_t *d_replica_offsets, float cutoff, float skin,
                                                        int32_t periodic, const float *box, int32_t *d_row_ptr,
                                                        int32_t *d_col, int32_t *d_rev, int64_t edge_capacity,
                                                        int64_t *d_n_edges, uint32_t *d_flags, void *cuda_stream);

/* Number of device kernels the library has launched on this context so far
 * (graph replays count each kernel node). */
SCHNET_API int64_t schnet_kernel_launches(const schnet_ctx *ctx);

#ifdef __cplusplus
}
#endif

#endif /* SCHNET_B200_H */
