// C ABI: context, workspace carving, weight packing, call orchestration and the
// per-rebuild-interval CUDA Graph.
//
// The step structure follows "Ab Initio Accuracy Beyond the Cutoff" (Tessera),
// abstract: with a conservative skin the neighbour graph and every tensor shape
// stay fixed between rebuilds, so one rebuild interval (build + n_rebuild
// steps of forward, backward and integration) is captured once and replayed as
// one CUDA Graph; the edge count stays on the device, so the host never reads
// data on the step path.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>

#include "internal.h"

using namespace schnet;

namespace {

constexpr int MAX_CTA = 1024;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Carver {
    uint8_t* base;
    size_t off = 0;
    template <class T>
    T* take(size_t count)
    {
        off = align_up(off, 256);
        T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
        off += std::max<size_t>(count, 1) * sizeof(T);
        return p;
    }
};

struct Derived {
    int N, R, T, F, K, L;
    int64_t cap;
    int ncell, nchunk;
    int gdim[3];
    double rl;
};

schnet_status validate(const schnet_config* c, std::string& why)
{
    if (!c) { why = "null config"; return SCHNET_ERR_INVALID_ARG; }
    if (c->n_types < 1) { why = "n_types < 1"; return SCHNET_ERR_INVALID_ARG; }
    if (c->n_features < 2 || c->n_features > FP || (c->n_features & 1)) {
        why = "n_features must be even and in [2, 128]";
        return SCHNET_ERR_UNSUPPORTED;
    }
    if (c->n_rbf < 1 || c->n_rbf > KP) { why = "n_rbf must be in [1, 64]"; return SCHNET_ERR_UNSUPPORTED; }
    if (c->n_interactions < 1 || c->n_interactions > MAX_L) {
        why = "n_interactions must be in [1, 8]";
        return SCHNET_ERR_UNSUPPORTED;
    }
    if (!(c->cutoff > 0.f) || !(c->skin >= 0.f) || !(c->rbf_sigma > 0.f) || !(c->rbf_max >= c->rbf_min)) {
        why = "cutoff/skin/rbf parameters out of range";
        return SCHNET_ERR_INVALID_ARG;
    }
    if (c->n_atoms < 1 || c->n_replicas < 1 || !c->replica_offsets) {
        why = "n_atoms, n_replicas and replica_offsets are required";
        return SCHNET_ERR_INVALID_ARG;
    }
    if (c->replica_offsets[0] != 0 || c->replica_offsets[c->n_replicas] != c->n_atoms) {
        why = "replica_offsets must start at 0 and end at n_atoms";
        return SCHNET_ERR_INVALID_ARG;
    }
    for (int r = 0; r < c->n_replicas; ++r)
        if (c->replica_offsets[r + 1] < c->replica_offsets[r]) {
            why = "replica_offsets must be non-decreasing";
            return SCHNET_ERR_INVALID_ARG;
        }
    if (c->periodic) {
        for (int d = 0; d < 3; ++d)
            if (!(c->box[d] >= 2.0f * (c->cutoff + c->skin))) {
                why = "periodic box must be at least 2 (cutoff + skin) in every dimension";
                return SCHNET_ERR_UNSUPPORTED;
            }
    }
    if (c->weight_dtype < 0 || c->weight_dtype > 3) { why = "weight_dtype"; return SCHNET_ERR_INVALID_ARG; }
    if ((int64_t)c->n_atoms * FP > (int64_t)1 << 40) { why = "too many atoms"; return SCHNET_ERR_UNSUPPORTED; }
    return SCHNET_OK;
}

Derived derive(const schnet_config* c)
{
    Derived d;
    d.N = c->n_atoms; d.R = c->n_replicas; d.T = c->n_types; d.F = c->n_features; d.K = c->n_rbf;
    d.L = c->n_interactions;
    d.rl = (double)c->cutoff + (double)c->skin;
    const double sphere = 4.0 / 3.0 * M_PI * d.rl * d.rl * d.rl;
    if (c->periodic) {
        long long cells = 1;
        for (int k = 0; k < 3; ++k) {
            const int g = cells_across((double)c->box[k], d.rl, GMAX_PERIODIC);
            d.gdim[k] = g;
            cells *= g;
        }
        d.ncell = (int)(cells * d.R);
    } else {
        d.gdim[0] = d.gdim[1] = d.gdim[2] = GMAX_NONPERIODIC;
        d.ncell = d.R * GMAX_NONPERIODIC * GMAX_NONPERIODIC * GMAX_NONPERIODIC;
    }
    d.nchunk = 0;
    int64_t cap = 0;
    for (int r = 0; r < d.R; ++r) {
        int64_t nr = c->replica_offsets[r + 1] - c->replica_offsets[r];
        d.nchunk += std::max<int64_t>(1, (nr + REDUCE_CHUNK - 1) / REDUCE_CHUNK);
        int64_t per;
        if (c->periodic) {
            double vol = (double)c->box[0] * c->box[1] * c->box[2];
            per = (int64_t)std::ceil(2.0 * sphere * (double)nr / vol) + 16;
        } else {
            per = (int64_t)std::ceil(sphere * 0.06) + 16;   // a dense bound for beads >= ~3 A apart
        }
        cap += nr * std::min<int64_t>(std::max<int64_t>(nr - 1, 0), per);
    }
    d.cap = c->edge_capacity > 0 ? c->edge_capacity : std::max<int64_t>(cap, 1);
    return d;
}

// Lays out every segment; with base == nullptr only measures.
size_t carve(const Derived& d, uint8_t* base, Workspace& w, size_t* wbegin = nullptr, size_t* wend = nullptr)
{
    Carver cv{base};
    const size_t N = d.N, L = d.L, R = d.R;
    w.meta = cv.take<DevMeta>(1);
    cv.off = align_up(cv.off, 256);
    if (wbegin) *wbegin = cv.off;
    w.img = cv.take<uint8_t>(L * LAYER_IMG);
    w.s1 = cv.take<float>(L * FP); w.s2 = cv.take<float>(L * FP);
    w.b1 = cv.take<float>(L * FP); w.b2 = cv.take<float>(L * FP);
    w.emb = cv.take<float>((size_t)d.T * FP);
    w.emb_h0 = cv.take<float>((size_t)d.T * FP);
    w.aw_img = cv.take<uint8_t>((size_t)(6 * L + 2) * AW_IMG);
    w.aw_sc = cv.take<float>((size_t)(6 * L + 2) * FP);
    w.bo1 = cv.take<float>(L * FP); w.bo2 = cv.take<float>(L * FP);
    w.c1 = cv.take<float>(HP); w.R2 = cv.take<float>(HP); w.c2 = cv.take<float>(4);
    w.rep_off = cv.take<int32_t>(R + 1);
    w.atom_rep = cv.take<int32_t>(N);
    w.chunk_rep = cv.take<int32_t>(d.nchunk); w.chunk_lo = cv.take<int32_t>(d.nchunk);
    w.chunk_hi = cv.take<int32_t>(d.nchunk);
    cv.off = align_up(cv.off, 256);
    if (wend) *wend = cv.off;
    w.pos4 = cv.take<float4>(N); w.ref4 = cv.take<float4>(N); w.frc4 = cv.take<float4>(N);
    w.perm = cv.take<int32_t>(N); w.cell_slot = cv.take<int32_t>(N);
    w.row_ptr = cv.take<int32_t>(N + 1); w.rowcnt = cv.take<int32_t>(N + 1);
    w.hcnt = cv.take<int32_t>(N + 1); w.rcnt = cv.take<int32_t>(N + 1);
    w.col = cv.take<int32_t>(d.cap); w.coltmp = cv.take<int32_t>(d.cap);
    w.rev = cv.take<int32_t>(d.cap); w.erow = cv.take<int32_t>(d.cap);
    w.s_edge = cv.take<float>(d.cap);
    w.crow = cv.take<int32_t>(d.cap); w.ccol = cv.take<int32_t>(d.cap); w.cidx = cv.take<int32_t>(d.cap);
    w.cdist = cv.take<float>(d.cap);
    w.ccount = cv.take<int32_t>(MAX_CTA);
    w.part = cv.take<int32_t>(MAX_CTA + 1);
    w.crow_h = cv.take<int32_t>(d.cap); w.ccol_h = cv.take<int32_t>(d.cap); w.cidx_h = cv.take<int32_t>(d.cap);
    w.cdist_h = cv.take<float>(d.cap);
    w.ccount_h = cv.take<int32_t>(MAX_CTA);
    w.part_h = cv.take<int32_t>(MAX_CTA + 1);
    w.crow_r = cv.take<int32_t>(d.cap); w.ccol_r = cv.take<int32_t>(d.cap); w.cdist_r = cv.take<float>(d.cap);
    w.ccount_r = cv.take<int32_t>(MAX_CTA);
    w.part_r = cv.take<int32_t>(MAX_CTA + 1);
    w.cell_of = cv.take<int32_t>(N); w.cell_atoms = cv.take<int32_t>(N);
    w.cell_cnt = cv.take<int32_t>((size_t)d.ncell + 1); w.cell_start = cv.take<int32_t>((size_t)d.ncell + 1);
    w.cell_fill = cv.take<int32_t>((size_t)d.ncell + 1);
    w.rgrid_dims = cv.take<int4>(R); w.rgrid_geom = cv.take<GridGeom>(R);
    w.scan_tmp = cv.take<long long>(SCAN_TILE);
    w.x = cv.take<float>(N * FP);
    w.h = cv.take<float>(L * N * FP);
    w.q = cv.take<float>(L * N * FP);
    w.m = cv.take<float>(N * FP); w.g = cv.take<float>(N * FP); w.dh = cv.take<float>(N * FP); w.dh2 = cv.take<float>(N * FP);
    w.pr = cv.take<float>(N * HP); w.eps = cv.take<float>(N); w.ke = cv.take<float>(N);
    w.partial = cv.take<double>(d.nchunk);
    w.epot = cv.take<double>(R); w.ekin = cv.take<double>(R);
    w.st_pos = cv.take<float>(3 * N); w.st_vel = cv.take<float>(3 * N); w.st_mass = cv.take<float>(N);
    w.st_types = cv.take<int32_t>(N);
    w.st_epot = cv.take<double>(R); w.st_ekin = cv.take<double>(R);
    return align_up(cv.off, 256);
}

// --- host packing of the filter-network weights --------------------------------
uint16_t to16(double v, int dtype_fmt)
{
    if (dtype_fmt == 1) return __bfloat16_as_ushort(__double2bfloat16(v));
    return __half_as_ushort(__double2half(v));
}
double from16(uint16_t u, int dtype_fmt)
{
    if (dtype_fmt == 1) return (double)__bfloat162float(__ushort_as_bfloat16(u));
    return (double)__half2float(__ushort_as_half(u));
}

// One [128 x KD] K-major A operand (rows = output channel f, K = input index k)
// of W[k][f] / s_f; two 16-bit terms when n_terms == 2.
void pack_operand(const float* W, int kin, int fout, int KD, const std::vector<double>& s, int fmt, int n_terms,
                  uint16_t* hi, uint16_t* lo)
{
    for (int f = 0; f < FP; ++f)
        for (int k = 0; k < KD; ++k) {
            double v = (f < fout && k < kin) ? (double)W[(size_t)k * fout + f] / s[f] : 0.0;
            uint16_t h = to16(v, fmt);
            uint16_t l = n_terms == 2 ? to16(v - from16(h, fmt), fmt) : (uint16_t)0;
            size_t idx = kmajor_off(f, k, FP) / 2;
            hi[idx] = h;
            lo[idx] = l;
        }
}

// An atom-wise dense layer as a tensor-core A operand for D[r][atom] = sum_k A[r][k] X[atom][k]:
// A[r][k] = W[k][r] (transposed use, y = x W) or W[r][k] (y = g W^T), W row-major [nrow][ncol],
// zero outside.  Each row r is divided by its max-abs s_r (1 for a zero row), stored as fp16
// hi + lo terms in the K-major core-matrix layout; s_r goes to sc[r].
void pack_aw(const float* W, int nrow, int ncol, bool transposed, uint8_t* img, float* sc)
{
    uint16_t* hi = reinterpret_cast<uint16_t*>(img);
    uint16_t* lo = reinterpret_cast<uint16_t*>(img + AW_IMG / 2);
    auto A = [&](int r, int k) -> double {
        if (transposed) return (k < nrow && r < ncol) ? (double)W[(size_t)k * ncol + r] : 0.0;
        return (r < nrow && k < ncol) ? (double)W[(size_t)r * ncol + k] : 0.0;
    };
    for (int r = 0; r < FP; ++r) {
        double m = 0.0;
        for (int k = 0; k < FP; ++k) m = std::max(m, std::fabs(A(r, k)));
        const float s = m > 0.0 ? (float)m : 1.0f;
        sc[r] = s;
        for (int k = 0; k < FP; ++k) {
            const double v = A(r, k) / (double)s;
            const uint16_t h = to16(v, 0);
            const size_t idx = kmajor_off(r, k, FP) / 2;
            hi[idx] = h;
            lo[idx] = to16(v - from16(h, 0), 0);
        }
    }
}

std::vector<double> channel_scales(const float* W, int kin, int fout)
{
    std::vector<double> s(FP, 1.0);
    for (int f = 0; f < fout; ++f) {
        double m = 0.0;
        for (int k = 0; k < kin; ++k) m = std::max(m, std::fabs((double)W[(size_t)k * fout + f]));
        s[f] = m > 0.0 ? m : 1.0;
    }
    return s;
}

void pad_mat(const float* src, int rin, int cin, float* dst, int rout, int cout_, bool transpose)
{
    for (int r = 0; r < rout; ++r)
        for (int c = 0; c < cout_; ++c) {
            float v = 0.f;
            if (!transpose) {
                if (r < rin && c < cin) v = src[(size_t)r * cin + c];
            } else {
                if (c < rin && r < cin) v = src[(size_t)c * cin + r];
            }
            dst[(size_t)r * cout_ + c] = v;
        }
}

void build_weight_blob(const schnet_ctx* c, const schnet_weights* wt, uint8_t* wsbase, uint8_t* blob,
                       size_t wbegin)
{
    const Workspace& w = c->ws;
    auto H = [&](auto* devp) { return reinterpret_cast<decltype(devp)>(blob + ((uint8_t*)devp - wsbase - wbegin)); };
    const int F = c->F, K = c->K, L = c->L, Hh = c->H;
    const int fmt = c->weight_fmt;
    for (int l = 0; l < L; ++l) {
        const float* W1 = wt->W1 + (size_t)l * K * F;
        const float* W2 = wt->W2 + (size_t)l * F * F;
        std::vector<double> s1 = channel_scales(W1, K, F), s2 = channel_scales(W2, F, F);
        uint8_t* img = H(w.img) + (size_t)l * LAYER_IMG;
        uint16_t* w1hi = reinterpret_cast<uint16_t*>(img);
        uint16_t* w1lo = reinterpret_cast<uint16_t*>(img + W1_IMG);
        uint16_t* w2hi = reinterpret_cast<uint16_t*>(img + 2 * W1_IMG);
        uint16_t* w2lo = reinterpret_cast<uint16_t*>(img + 2 * W1_IMG + W2_IMG);
        pack_operand(W1, K, F, KP, s1, fmt, c->n_wterms, w1hi, w1lo);
        pack_operand(W2, F, F, FP, s2, fmt, c->n_wterms, w2hi, w2lo);
        // With one 16-bit activation term the kernels feed the second layer
        // a = log2(1 + e^x) = ssp(x) / ln2 + 1 (see the forward epilogue): the -1 goes
        // into the bias as -ln2 s2 times the column sum of the stored weight terms.
        std::vector<double> colsum(FP, 0.0);
        if (c->n_xterms == 1)
            for (int f = 0; f < FP; ++f)
                for (int k = 0; k < FP; ++k) {
                    const size_t idx = kmajor_off(f, k, FP) / 2;
                    colsum[f] += from16(w2hi[idx], fmt) + (c->n_wterms == 2 ? from16(w2lo[idx], fmt) : 0.0);
                }
        for (int f = 0; f < FP; ++f) {
            H(w.s1)[l * FP + f] = (float)s1[f];
            H(w.s2)[l * FP + f] = (float)s2[f];
            H(w.b1)[l * FP + f] = f < F ? wt->b1[l * F + f] : 0.f;
            const double b2 = f < F ? (double)wt->b2[l * F + f] : 0.0;
            H(w.b2)[l * FP + f] = (float)(b2 - 0.69314718055994530942 * s2[f] * colsum[f]);
            H(w.bo1)[l * FP + f] = f < F ? wt->bo1[l * F + f] : 0.f;
            H(w.bo2)[l * FP + f] = f < F ? wt->bo2[l * F + f] : 0.f;
        }
        const size_t oi = (size_t)l * F * F;
        const float* mats[6] = {wt->Wo1 + oi, wt->Wo2 + oi, wt->W_in + oi, wt->W_in + oi, wt->Wo2 + oi, wt->Wo1 + oi};
        for (int j = 0; j < 6; ++j)
            pack_aw(mats[j], F, F, j < 3, H(w.aw_img) + (size_t)(6 * l + j) * AW_IMG, H(w.aw_sc) + (size_t)(6 * l + j) * FP);
    }
    pack_aw(wt->R1, F, Hh, true, H(w.aw_img) + (size_t)(6 * L) * AW_IMG, H(w.aw_sc) + (size_t)(6 * L) * FP);
    pack_aw(wt->R1, F, Hh, false, H(w.aw_img) + (size_t)(6 * L + 1) * AW_IMG, H(w.aw_sc) + (size_t)(6 * L + 1) * FP);
    pad_mat(wt->emb, c->T, F, H(w.emb), c->T, FP, false);
    // x0 = emb[z] has one row per type, so h0 = x0 W_in of interaction 0 does too (float64 sums)
    for (int t = 0; t < c->T; ++t)
        for (int f = 0; f < FP; ++f) {
            double acc = 0.0;
            if (f < F)
                for (int k = 0; k < F; ++k) acc += (double)wt->emb[(size_t)t * F + k] * (double)wt->W_in[(size_t)k * F + f];
            H(w.emb_h0)[(size_t)t * FP + f] = (float)acc;
        }
    for (int k = 0; k < HP; ++k) {
        H(w.c1)[k] = k < Hh ? wt->c1[k] : 0.f;
        H(w.R2)[k] = k < Hh ? wt->R2[k] : 0.f;
    }
    H(w.c2)[0] = wt->c2;
    // replica tables
    for (int r = 0; r <= c->R; ++r) H(w.rep_off)[r] = c->rep_off[r];
    int32_t* ar = H(w.atom_rep);
    int ch = 0;
    for (int r = 0; r < c->R; ++r) {
        int a = c->rep_off[r], b = c->rep_off[r + 1];
        for (int i = a; i < b; ++i) ar[i] = r;
        int nr = b - a;
        int nch = std::max(1, (nr + REDUCE_CHUNK - 1) / REDUCE_CHUNK);
        for (int k = 0; k < nch; ++k, ++ch) {
            H(w.chunk_rep)[ch] = r;
            H(w.chunk_lo)[ch] = std::min(b, a + k * REDUCE_CHUNK);
            H(w.chunk_hi)[ch] = std::min(b, a + (k + 1) * REDUCE_CHUNK);
        }
    }
}

schnet_status fail(schnet_ctx* c, schnet_status st, const std::string& msg)
{
    if (c) c->err = msg;
    return st;
}

schnet_status cuda_fail(schnet_ctx* c, cudaError_t e, const char* where)
{
    return fail(c, SCHNET_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

#define CK(expr)                                                   \
    do {                                                           \
        cudaError_t e_ = (expr);                                   \
        if (e_ != cudaSuccess) return cuda_fail(c, e_, #expr);     \
    } while (0)

// Event pair around one launch on the library stream while profiling.
struct Timed {
    schnet_ctx* c;
    int kind;
    cudaEvent_t a = nullptr, b = nullptr;
    Timed(schnet_ctx* c_, int k) : c(c_), kind(k)
    {
        if (c->prof && cudaEventCreate(&a) == cudaSuccess) cudaEventRecord(a, c->s);
    }
    ~Timed()
    {
        if (c->prof && a && cudaEventCreate(&b) == cudaSuccess) {
            cudaEventRecord(b, c->s);
            c->prof_pairs[kind].push_back({a, b});
        }
    }
};

void join_in(schnet_ctx* c)
{
    cudaEventRecord(c->ev_in, c->user_stream);
    cudaStreamWaitEvent(c->s, c->ev_in, 0);
}

cudaError_t join_out(schnet_ctx* c)
{
    cudaError_t e = cudaEventRecord(c->ev_out, c->s);
    if (e != cudaSuccess) return e;
    return cudaStreamWaitEvent(c->user_stream, c->ev_out, 0);
}

schnet_status status_from_flags(unsigned int f)
{
    if (f & SCHNET_FLAG_TIMEOUT) return SCHNET_ERR_TIMEOUT;
    if (f & SCHNET_FLAG_CAPACITY) return SCHNET_ERR_CAPACITY;
    if (f & SCHNET_FLAG_BADTYPE) return SCHNET_ERR_BADTYPE;
    if (f & SCHNET_FLAG_NONFINITE) return SCHNET_ERR_NONFINITE;
    if (f & SCHNET_FLAG_SKIN) return SCHNET_ERR_SKIN;
    return SCHNET_OK;
}

cudaError_t read_and_clear_flags(schnet_ctx* c, unsigned int* flags)
{
    DevMeta hm;
    cudaError_t e = cudaMemcpyAsync(&hm, c->ws.meta, sizeof(DevMeta), cudaMemcpyDeviceToHost, c->s);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(&c->ws.meta->status, 0, sizeof(unsigned int), c->s);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(c->s);
    *flags = hm.status;
    return e;
}

// k MD steps, optionally preceded by a neighbour build at the current positions.
// The per-replica potential and kinetic energies are summed at the last of the k
// steps only: they are returned for the last step of a call, and a call's steps
// end at the end of an enqueued block.
cudaError_t enqueue_steps(schnet_ctx* c, int k, bool build_first, float* pos, float* vel, const int32_t* types,
                          const float* mass, const schnet_step_params* p, double* epot, double* ekin)
{
    cudaError_t e;
    if (build_first) {
        Timed t(c, SCHNET_KERNEL_NEIGHBORS);
        if ((e = launch_build_neighbors(c, pos)) != cudaSuccess) return e;
    }
    for (int s = 0; s < k; ++s) {
        {
            Timed t(c, SCHNET_KERNEL_INTEGRATE);
            if ((e = launch_baoa(c, pos, vel, mass, p->dt_fs, p->gamma_per_ps, p->temperature_K, p->seed,
                                 p->d_noise, true)) != cudaSuccess)
                return e;
        }
        const bool last = s == k - 1;
        if ((e = launch_energy_forces(c, types, epot, nullptr, true, last)) != cudaSuccess) return e;
        {
            Timed t(c, SCHNET_KERNEL_INTEGRATE);
            if ((e = launch_b_kick(c, vel, mass, p->dt_fs, ekin, last)) != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

// Run `k` steps (with a build first if asked) as a cached CUDA Graph, or eagerly.
schnet_status run_steps(schnet_ctx* c, int slot, int k, bool build_first, const GraphKey& key, float* pos,
                        float* vel, const int32_t* types, const float* mass, const schnet_step_params* p,
                        double* ep, double* ek)
{
    if (!p->use_graph) {
        CK(enqueue_steps(c, k, build_first, pos, vel, types, mass, p, ep, ek));
        return SCHNET_OK;
    }
    auto& g = c->graphs[slot];
    if (!g.ok || !(key == g.key)) {
        if (g.exec) { cudaGraphExecDestroy(g.exec); g.exec = nullptr; }
        g.ok = false;
        int64_t before = c->launches;
        CK(cudaStreamBeginCapture(c->s, cudaStreamCaptureModeThreadLocal));
        cudaError_t ce = enqueue_steps(c, k, build_first, pos, vel, types, mass, p, ep, ek);
        cudaGraph_t graph = nullptr;
        cudaError_t ee = cudaStreamEndCapture(c->s, &graph);
        g.kernels = c->launches - before;   // kernels captured per replay
        c->launches = before;
        if (ce != cudaSuccess) { if (graph) cudaGraphDestroy(graph); return cuda_fail(c, ce, "capture"); }
        if (ee != cudaSuccess) return cuda_fail(c, ee, "cudaStreamEndCapture");
        cudaError_t ie = cudaGraphInstantiate(&g.exec, graph, 0);
        cudaGraphDestroy(graph);
        if (ie != cudaSuccess) return cuda_fail(c, ie, "cudaGraphInstantiate");
        g.key = key;
        g.ok = true;
    }
    CK(cudaGraphLaunch(g.exec, c->s));
    c->launches += g.kernels;
    return SCHNET_OK;
}

// The list is rebuilt before the first step of every interval of n_rebuild
// steps; the phase persists across calls with resume = 1.  Aligned full
// intervals replay one graph each; other steps replay single-step graphs.
schnet_status step_impl(schnet_ctx* c, float* pos, float* vel, const int32_t* types, const float* mass,
                        int64_t n_steps, const schnet_step_params* p, double* epot, double* ekin)
{
    if (!pos || !vel || !types || !mass || !p || n_steps < 0 || p->n_rebuild < 1 || !(p->dt_fs > 0.f) ||
        !(p->gamma_per_ps >= 0.f))
        return fail(c, SCHNET_ERR_INVALID_ARG, "schnet_step: bad argument");
    double* ep = epot ? epot : c->ws.epot;
    double* ek = ekin ? ekin : c->ws.ekin;
    if (!p->resume || !c->forces_valid) {
        c->have_list = false;            // fresh start: the build below replaces the list
        CK(launch_build_neighbors(c, pos));
        c->have_list = true;
        CK(launch_energy_forces(c, types, ep, nullptr, true));
        c->since_build = p->n_rebuild;   // the first interval starts with a fresh build
    }
    if (c->since_build > p->n_rebuild) c->since_build = p->n_rebuild;
    CK(launch_set_step(c, p->step0));
    GraphKey key{pos, vel, types, mass, ep, ek, p->d_noise, p->dt_fs, p->gamma_per_ps, p->temperature_K,
                 p->n_rebuild, (unsigned long long)p->seed};
    int64_t left = n_steps;
    schnet_status st;
    while (left > 0) {
        const bool need_build = c->since_build >= p->n_rebuild;
        if (need_build && left >= p->n_rebuild) {
            if ((st = run_steps(c, 0, p->n_rebuild, true, key, pos, vel, types, mass, p, ep, ek)) != SCHNET_OK)
                return st;
            c->since_build = p->n_rebuild;
            left -= p->n_rebuild;
        } else {
            if ((st = run_steps(c, need_build ? 1 : 2, 1, need_build, key, pos, vel, types, mass, p, ep, ek)) !=
                SCHNET_OK)
                return st;
            c->since_build = need_build ? 1 : c->since_build + 1;
            left -= 1;
        }
    }
    c->forces_valid = true;
    return SCHNET_OK;
}

}  // namespace

// ============================================================================
// energy / forces orchestration
// ============================================================================
// need_forces = false: energies only (no backward, internal forces left as they were);
// sum_energy = false: per-atom energies only, no per-replica sums
cudaError_t schnet::launch_energy_forces(schnet_ctx* c, const int32_t* types, double* energy, float* forces,
                                         bool need_forces, bool sum_energy)
{
    cudaError_t e;
#define SCHNET_TIMED(kind, expr)                        \
    do {                                                \
        Timed t_(c, kind);                              \
        if ((e = (expr)) != cudaSuccess) return e;      \
    } while (0)
    SCHNET_TIMED(SCHNET_KERNEL_MASK, launch_compact(c, need_forces));
    SCHNET_TIMED(SCHNET_KERNEL_ATOMWISE, launch_embed(c, types));
    for (int l = 0; l < c->L; ++l) {
        SCHNET_TIMED(SCHNET_KERNEL_CFCONV_FWD, launch_cfconv_fwd(c, l));
        SCHNET_TIMED(SCHNET_KERNEL_ATOMWISE, launch_aw_fwd(c, l));
    }
    if (sum_energy)
        SCHNET_TIMED(SCHNET_KERNEL_REDUCE, launch_replica_sum(c, c->ws.eps, energy ? energy : c->ws.epot));
    if (!need_forces) return cudaSuccess;
    SCHNET_TIMED(SCHNET_KERNEL_ATOMWISE, launch_aw_bwd_top(c));
    for (int l = c->L - 1; l >= 0; --l) {
        // pair derivatives over the half list (one edge per unordered pair) and, but for
        // interaction 0 (whose dE/dh would only reach the embedding, which forces do not
        // need), the half list's terms of dE/dh; the complementary list's launch forms the
        // rest, and the atom-wise backward adds the two and carries the gradient to the
        // earlier interactions
        SCHNET_TIMED(SCHNET_KERNEL_CFCONV_BWD, launch_cfconv_pair(c, l, l < c->L - 1 ? 1 : 0, l > 0));
        if (l > 0) {
            SCHNET_TIMED(SCHNET_KERNEL_CFCONV_DH, launch_cfconv_dh(c, l));
            SCHNET_TIMED(SCHNET_KERNEL_ATOMWISE, launch_aw_bwd(c, l));
        }
    }
    SCHNET_TIMED(SCHNET_KERNEL_FORCES, launch_forces(c, forces));
#undef SCHNET_TIMED
    return cudaSuccess;
}

// ============================================================================
// C ABI
// ============================================================================
extern "C" {

schnet_status schnet_workspace_bytes(const schnet_config* cfg, size_t* bytes)
{
    std::string why;
    if (!bytes) return SCHNET_ERR_INVALID_ARG;
    schnet_status st = validate(cfg, why);
    if (st != SCHNET_OK) return st;
    Derived d = derive(cfg);
    Workspace w;
    *bytes = carve(d, nullptr, w);
    return SCHNET_OK;
}

schnet_status schnet_create(const schnet_config* cfg, const schnet_weights* wt, void* cuda_stream,
                            void* d_workspace, size_t ws_bytes, schnet_ctx** out)
{
    if (!out) return SCHNET_ERR_INVALID_ARG;
    *out = nullptr;
    std::string why;
    schnet_status st = validate(cfg, why);
    if (st != SCHNET_OK) return st;
    if (!wt || !wt->emb || !wt->W_in || !wt->W1 || !wt->b1 || !wt->W2 || !wt->b2 || !wt->Wo1 || !wt->bo1 ||
        !wt->Wo2 || !wt->bo2 || !wt->R1 || !wt->c1 || !wt->R2)
        return SCHNET_ERR_INVALID_ARG;
    if (!d_workspace || ((uintptr_t)d_workspace & 255)) return SCHNET_ERR_INVALID_ARG;
    Derived d = derive(cfg);
    Workspace probe;
    size_t need = carve(d, nullptr, probe);
    if (ws_bytes < need) return SCHNET_ERR_INVALID_ARG;

    schnet_ctx* c = new (std::nothrow) schnet_ctx();
    if (!c) return SCHNET_ERR_INVALID_ARG;
    c->cfg = *cfg;
    c->rep_off.assign(cfg->replica_offsets, cfg->replica_offsets + cfg->n_replicas + 1);
    c->cfg.replica_offsets = nullptr;
    c->N = d.N; c->R = d.R; c->T = d.T; c->F = d.F; c->K = d.K; c->L = d.L; c->H = d.F / 2;
    c->weight_fmt = cfg->weight_dtype == SCHNET_WEIGHTS_BF16 ? 1 : 0;
    c->n_wterms = cfg->weight_dtype == SCHNET_WEIGHTS_FP32 ? 2 : 1;
    c->n_xterms = cfg->weight_dtype == SCHNET_WEIGHTS_FP16_FAST ? 1 : 2;
    c->cap = d.cap;
    c->ncell = d.ncell;
    c->nchunk = d.nchunk;
    for (int k = 0; k < 3; ++k) c->gdim[k] = d.gdim[k];
    c->rl2 = d.rl * d.rl;
    c->mu0 = cfg->rbf_min;
    c->dmu = d.K > 1 ? (float)(((double)cfg->rbf_max - (double)cfg->rbf_min) / (double)(d.K - 1)) : 0.f;
    c->box.periodic = cfg->periodic;
    for (int k = 0; k < 3; ++k) {
        c->box.L[k] = cfg->periodic ? cfg->box[k] : 0.f;
        c->box.invL[k] = cfg->periodic ? 1.0f / cfg->box[k] : 0.f;
    }
    c->user_stream = (cudaStream_t)cuda_stream;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->s, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_in, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_out, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cfconv_init_attributes();
    if (e == cudaSuccess) e = atomwise_init_attributes();
    if (e != cudaSuccess) {
        delete c;
        return SCHNET_ERR_CUDA;
    }
    c->ncta = std::min(c->nsm, MAX_CTA);

    size_t wbegin = 0, wend = 0;
    uint8_t* base = (uint8_t*)d_workspace;
    carve(d, base, c->ws, &wbegin, &wend);
    std::vector<uint8_t> blob(wend - wbegin, 0);
    build_weight_blob(c, wt, base, blob.data(), wbegin);
    join_in(c);
    e = cudaMemcpyAsync(base + wbegin, blob.data(), blob.size(), cudaMemcpyHostToDevice, c->s);
    if (e == cudaSuccess) e = cudaMemsetAsync(c->ws.meta, 0, sizeof(DevMeta), c->s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(c->s);
    if (e != cudaSuccess) {
        schnet_destroy(c);
        return SCHNET_ERR_CUDA;
    }
    *out = c;
    return SCHNET_OK;
}

schnet_status schnet_build_neighbors(schnet_ctx* c, const float* d_pos)
{
    if (!c || !d_pos) return SCHNET_ERR_INVALID_ARG;
    join_in(c);
    c->have_list = false;
    CK(launch_build_neighbors(c, d_pos));
    c->have_list = true;
    c->forces_valid = false;
    CK(join_out(c));
    return SCHNET_OK;
}

schnet_status schnet_energy_forces(schnet_ctx* c, const float* d_pos, const int32_t* d_types, double* d_energy,
                                   float* d_forces)
{
    if (!c || !d_pos || !d_types || !d_energy) return SCHNET_ERR_INVALID_ARG;
    if (!c->have_list) return fail(c, SCHNET_ERR_STATE, "schnet_energy_forces: build the neighbour list first");
    join_in(c);
    CK(launch_pack_positions(c, d_pos));
    CK(launch_energy_forces(c, d_types, d_energy, d_forces, d_forces != nullptr));
    c->forces_valid = false;
    CK(join_out(c));
    return SCHNET_OK;
}

schnet_status schnet_step(schnet_ctx* c, float* d_pos, float* d_vel, const int32_t* d_types, const float* d_mass,
                          int64_t n_steps, const schnet_step_params* p, double* d_epot, double* d_ekin)
{
    if (!c) return SCHNET_ERR_INVALID_ARG;
    join_in(c);
    schnet_status st = step_impl(c, d_pos, d_vel, d_types, d_mass, n_steps, p, d_epot, d_ekin);
    if (st != SCHNET_OK) return st;
    unsigned int flags = 0;
    CK(join_out(c));
    CK(read_and_clear_flags(c, &flags));
    return status_from_flags(flags);
}

schnet_status schnet_step_host(schnet_ctx* c, float* h_pos, float* h_vel, const int32_t* h_types,
                               const float* h_mass, int64_t n_steps, const schnet_step_params* p, double* h_epot,
                               double* h_ekin)
{
    if (!c || !h_pos || !h_vel || !h_types || !h_mass) return SCHNET_ERR_INVALID_ARG;
    Workspace& w = c->ws;
    const size_t N = c->N, R = c->R;
    join_in(c);
    CK(cudaMemcpyAsync(w.st_pos, h_pos, 3 * N * sizeof(float), cudaMemcpyHostToDevice, c->s));
    CK(cudaMemcpyAsync(w.st_vel, h_vel, 3 * N * sizeof(float), cudaMemcpyHostToDevice, c->s));
    CK(cudaMemcpyAsync(w.st_types, h_types, N * sizeof(int32_t), cudaMemcpyHostToDevice, c->s));
    CK(cudaMemcpyAsync(w.st_mass, h_mass, N * sizeof(float), cudaMemcpyHostToDevice, c->s));
    schnet_status st = step_impl(c, w.st_pos, w.st_vel, w.st_types, w.st_mass, n_steps, p, w.st_epot, w.st_ekin);
    if (st != SCHNET_OK) return st;
    CK(cudaMemcpyAsync(h_pos, w.st_pos, 3 * N * sizeof(float), cudaMemcpyDeviceToHost, c->s));
    CK(cudaMemcpyAsync(h_vel, w.st_vel, 3 * N * sizeof(float), cudaMemcpyDeviceToHost, c->s));
    if (h_epot) CK(cudaMemcpyAsync(h_epot, w.st_epot, R * sizeof(double), cudaMemcpyDeviceToHost, c->s));
    if (h_ekin) CK(cudaMemcpyAsync(h_ekin, w.st_ekin, R * sizeof(double), cudaMemcpyDeviceToHost, c->s));
    unsigned int flags = 0;
    CK(join_out(c));
    CK(read_and_clear_flags(c, &flags));
    return status_from_flags(flags);
}

schnet_status schnet_get_status(schnet_ctx* c, uint32_t* flags)
{
    if (!c || !flags) return SCHNET_ERR_INVALID_ARG;
    join_in(c);
    unsigned int f = 0;
    CK(read_and_clear_flags(c, &f));
    *flags = f;
    return SCHNET_OK;
}

const char* schnet_last_error(const schnet_ctx* c) { return c ? c->err.c_str() : "null context"; }

schnet_status schnet_destroy(schnet_ctx* c)
{
    if (!c) return SCHNET_OK;
    if (c->s) cudaStreamSynchronize(c->s);
    for (auto& g : c->graphs)
        if (g.exec) cudaGraphExecDestroy(g.exec);
    if (c->ev_in) cudaEventDestroy(c->ev_in);
    if (c->ev_out) cudaEventDestroy(c->ev_out);
    if (c->s) cudaStreamDestroy(c->s);
    delete c;
    return SCHNET_OK;
}

schnet_status schnet_get_neighbors(schnet_ctx* c, int32_t* h_row_ptr, int32_t* h_col, int32_t* h_rev,
                                   int64_t* n_edges, int64_t cap)
{
    if (!c) return SCHNET_ERR_INVALID_ARG;
    if (!c->have_list) return fail(c, SCHNET_ERR_STATE, "no neighbour list");
    join_in(c);
    DevMeta hm;
    CK(cudaMemcpyAsync(&hm, c->ws.meta, sizeof(DevMeta), cudaMemcpyDeviceToHost, c->s));
    CK(cudaStreamSynchronize(c->s));
    if (n_edges) *n_edges = hm.n_edges;
    if (hm.n_edges > c->cap) return fail(c, SCHNET_ERR_CAPACITY, "edge list overflowed its capacity");
    if ((h_col || h_rev) && cap < hm.n_edges) return fail(c, SCHNET_ERR_CAPACITY, "host buffer too small");
    const int32_t *rp = nullptr, *col = nullptr, *rev = nullptr;
    CK(launch_caller_order_list(c, &rp, &col, &rev));
    if (h_row_ptr) CK(cudaMemcpyAsync(h_row_ptr, rp, (c->N + 1) * sizeof(int32_t), cudaMemcpyDeviceToHost, c->s));
    if (h_col) CK(cudaMemcpyAsync(h_col, col, hm.n_edges * sizeof(int32_t), cudaMemcpyDeviceToHost, c->s));
    if (h_rev) CK(cudaMemcpyAsync(h_rev, rev, hm.n_edges * sizeof(int32_t), cudaMemcpyDeviceToHost, c->s));
    CK(cudaStreamSynchronize(c->s));
    return SCHNET_OK;
}

schnet_status schnet_get_atom_energies(schnet_ctx* c, float* d_eps)
{
    if (!c || !d_eps) return SCHNET_ERR_INVALID_ARG;
    if (!c->have_list) return fail(c, SCHNET_ERR_STATE, "no neighbour list");
    join_in(c);
    CK(launch_scatter_atoms(c, c->ws.eps, d_eps));
    CK(join_out(c));
    return SCHNET_OK;
}

schnet_status schnet_profile_steps(schnet_ctx* c, float* d_pos, float* d_vel, const int32_t* d_types,
                                   const float* d_mass, int64_t n_steps, const schnet_step_params* p,
                                   double* ms_total, int64_t* launches)
{
    if (!c || !p || !ms_total || !launches) return SCHNET_ERR_INVALID_ARG;
    schnet_step_params q = *p;
    q.use_graph = 0;
    join_in(c);
    if (!q.resume || !c->forces_valid) {
        schnet_status st0 = step_impl(c, d_pos, d_vel, d_types, d_mass, 0, &q, nullptr, nullptr);
        if (st0 != SCHNET_OK) return st0;
        q.resume = 1;
    }
    for (auto& v : c->prof_pairs) v.clear();
    c->prof = true;
    schnet_status st = step_impl(c, d_pos, d_vel, d_types, d_mass, n_steps, &q, nullptr, nullptr);
    c->prof = false;
    cudaError_t e = cudaStreamSynchronize(c->s);
    for (int k = 0; k < SCHNET_KERNEL_NCLASS; ++k) {
        double sum = 0.0;
        for (auto& pr : c->prof_pairs[k]) {
            float ms = 0.f;
            if (e == cudaSuccess && cudaEventElapsedTime(&ms, pr.first, pr.second) == cudaSuccess) sum += ms;
            cudaEventDestroy(pr.first);
            cudaEventDestroy(pr.second);
        }
        ms_total[k] = sum;
        launches[k] = (int64_t)c->prof_pairs[k].size();
        c->prof_pairs[k].clear();
    }
    if (st != SCHNET_OK) return st;
    if (e != cudaSuccess) return cuda_fail(c, e, "profile sync");
    unsigned int flags = 0;
    CK(join_out(c));
    CK(read_and_clear_flags(c, &flags));
    return status_from_flags(flags);
}

schnet_status schnet_test_timeout(schnet_ctx* c, uint32_t max_polls, int32_t complete)
{
    if (!c || max_polls < 1) return SCHNET_ERR_INVALID_ARG;
    join_in(c);
    CK(launch_test_timeout(c, max_polls, complete ? 1 : 0));
    CK(join_out(c));
    return SCHNET_OK;
}

int64_t schnet_kernel_launches(const schnet_ctx* c) { return c ? c->launches : 0; }

}  // extern "C"
