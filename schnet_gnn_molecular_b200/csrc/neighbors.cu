// Neighbour build: cell list -> destination-sorted CSR with skin, its
// transpose map rev[], and the per-CTA row partition of the tensor-core kernels.
//
// Follows "Ab Initio Accuracy Beyond the Cutoff" (Tessera), abstract: a
// conservative neighbour skin (list radius r_c + skin) keeps the graph valid
// between rebuilds; and FlashSchNet (paper-curation summary), How / flash
// aggregation: a CSR layout that lets every reduction run per row without
// atomics.  The pair test is done in float64 with every operation rounded on
// its own, so the list is a bit-exact function of the float32 coordinates.
#include <cmath>
#include <mutex>

#include "internal.h"

namespace schnet {

// ---------------------------------------------------------------------------
// exclusive scan (int32 in, int32 out, int64 total) -- three passes
// ---------------------------------------------------------------------------
__device__ __forceinline__ long long warp_incl_scan(long long v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        long long t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// block-wide exclusive scan of one value per thread; returns the block total
__device__ __forceinline__ long long block_excl_scan(long long v, long long& excl)
{
    __shared__ long long wsum[32];
    __shared__ long long wtotal;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    long long inc = warp_incl_scan(v);
    if (lane == 31) wsum[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        const int nw = blockDim.x >> 5;
        long long w = lane < nw ? wsum[lane] : 0;
        long long wi = warp_incl_scan(w);
        if (lane < nw) wsum[lane] = wi - w;   // exclusive prefix of each warp
        if (lane == nw - 1) wtotal = wi;      // block total
    }
    __syncthreads();
    excl = inc - v + wsum[wid];
    long long total = wtotal;
    __syncthreads();
    return total;
}

__global__ void k_scan_tiles(const int32_t* __restrict__ in, int n, long long* __restrict__ tile_sums)
{
    const int base = blockIdx.x * SCAN_TILE;
    long long s = 0;
#pragma unroll
    for (int k = 0; k < SCAN_ITEMS; ++k) {
        int i = base + threadIdx.x * SCAN_ITEMS + k;
        if (i < n) s += in[i];
    }
    long long ex;
    long long tot = block_excl_scan(s, ex);
    if (threadIdx.x == 0) tile_sums[blockIdx.x] = tot;
}

__global__ void k_scan_sums(long long* __restrict__ tile_sums, int ntiles)
{
    // one block of SCAN_BLOCK threads, ntiles <= SCAN_TILE
    long long v[SCAN_ITEMS];
    long long s = 0;
#pragma unroll
    for (int k = 0; k < SCAN_ITEMS; ++k) {
        int i = threadIdx.x * SCAN_ITEMS + k;
        v[k] = i < ntiles ? tile_sums[i] : 0;
        s += v[k];
    }
    long long ex;
    block_excl_scan(s, ex);
#pragma unroll
    for (int k = 0; k < SCAN_ITEMS; ++k) {
        int i = threadIdx.x * SCAN_ITEMS + k;
        if (i < ntiles) tile_sums[i] = ex;
        ex += v[k];
    }
}

// out[i] = exclusive prefix, out[n] = total (clamped to int32); *total64 = total
__global__ void k_scan_apply(const int32_t* __restrict__ in, int n, const long long* __restrict__ tile_sums,
                             int32_t* __restrict__ out, long long* total64, int ntiles)
{
    const int base = blockIdx.x * SCAN_TILE;
    long long v[SCAN_ITEMS];
    long long s = 0;
#pragma unroll
    for (int k = 0; k < SCAN_ITEMS; ++k) {
        int i = base + threadIdx.x * SCAN_ITEMS + k;
        v[k] = i < n ? in[i] : 0;
        s += v[k];
    }
    long long ex;
    block_excl_scan(s, ex);
    ex += tile_sums[blockIdx.x];
#pragma unroll
    for (int k = 0; k < SCAN_ITEMS; ++k) {
        int i = base + threadIdx.x * SCAN_ITEMS + k;
        if (i < n) out[i] = (int32_t)(ex < 0x7fffffffLL ? ex : 0x7fffffffLL);
        ex += v[k];
    }
    if (blockIdx.x == ntiles - 1 && threadIdx.x == blockDim.x - 1) {
        out[n] = (int32_t)(ex < 0x7fffffffLL ? ex : 0x7fffffffLL);
        if (total64) *total64 = ex;
    }
}

static cudaError_t scan_exclusive(schnet_ctx* c, const int32_t* in, int n, int32_t* out, long long* total64)
{
    int ntiles = (n + SCAN_TILE - 1) / SCAN_TILE;
    if (ntiles < 1) ntiles = 1;
    if (ntiles > SCAN_TILE) return cudaErrorInvalidValue;
    k_scan_tiles<<<ntiles, SCAN_BLOCK, 0, c->s>>>(in, n, c->ws.scan_tmp);
    k_scan_sums<<<1, SCAN_BLOCK, 0, c->s>>>(c->ws.scan_tmp, ntiles);
    k_scan_apply<<<ntiles, SCAN_BLOCK, 0, c->s>>>(in, n, c->ws.scan_tmp, out, total64, ntiles);
    c->launches += 3;
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// positions
//
// Between two builds every per-atom array of the energy / force path is held in
// "slot" order: atoms sorted by cell (cells grouped by replica, raster order
// inside a replica, ascending atom index inside a cell).  Atoms that are close
// in space are then close in memory, so the per-edge gathers of neighbour
// features hit cache lines and L2 sets that the neighbouring rows have just
// used.  perm[k] is the caller's index of the atom in slot k.  Positions,
// velocities, masses, forces and per-replica results stay in the caller's order.
// ---------------------------------------------------------------------------
__global__ void k_pack_positions(int n, const float* __restrict__ pos, const int32_t* __restrict__ perm,
                                 float4* __restrict__ pos4, const float4* __restrict__ ref4, int check_skin,
                                 float half_skin2, DevMeta* meta)
{
    int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= n) return;
    const int i = perm ? perm[k] : k;
    float x = pos[3 * i], y = pos[3 * i + 1], z = pos[3 * i + 2];
    pos4[k] = make_float4(x, y, z, 0.0f);
    if (!(isfinite(x) && isfinite(y) && isfinite(z))) set_flag(meta, SCHNET_FLAG_NONFINITE);
    if (check_skin) {
        float4 r = ref4[k];
        float dx = x - r.x, dy = y - r.y, dz = z - r.z;
        if (dx * dx + dy * dy + dz * dz > half_skin2) set_flag(meta, SCHNET_FLAG_SKIN);
    }
}

// caller positions -> slot order, with the skin check against the last build
cudaError_t launch_pack_positions(schnet_ctx* c, const float* d_pos)
{
    if (!c->have_list) return cudaErrorInvalidValue;
    float hs = 0.5f * c->cfg.skin;
    k_pack_positions<<<(c->N + 255) / 256, 256, 0, c->s>>>(c->N, d_pos, c->ws.perm, c->ws.pos4, c->ws.ref4, 1,
                                                            hs * hs, c->ws.meta);
    c->launches += 1;
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// cell grid per replica
// ---------------------------------------------------------------------------
struct GridParams {
    int periodic;
    int gp[3];          // periodic grid dims
    double rl;          // list radius r_c + skin
    int gmax;           // non-periodic max dims
    int cells_per_rep;  // stride between replicas' cell ranges
};

// One block per replica: grid dims and placement.  Periodic: the box's grid.
// Open boundaries: the replica's bounding box, split into cells_across() cells
// per dimension (at least r_c + skin wide, at most gmax per dimension).
__global__ void k_replica_grid(int R, const int32_t* __restrict__ rep_off, const float4* __restrict__ pos4,
                               GridParams gp, const Box box, int4* __restrict__ dims, GridGeom* __restrict__ geom)
{
    int r = blockIdx.x;
    if (r >= R) return;
    int a = rep_off[r], b = rep_off[r + 1];
    if (gp.periodic) {
        if (threadIdx.x == 0) {
            dims[r] = make_int4(gp.gp[0], gp.gp[1], gp.gp[2], r * gp.cells_per_rep);
            GridGeom gm;
            for (int d = 0; d < 3; ++d) {
                gm.org[d] = 0.0;
                gm.inv[d] = (double)gp.gp[d] / (double)box.L[d];
            }
            geom[r] = gm;
        }
        return;
    }
    float lo[3] = {3.4e38f, 3.4e38f, 3.4e38f}, hi[3] = {-3.4e38f, -3.4e38f, -3.4e38f};
    for (int i = a + threadIdx.x; i < b; i += blockDim.x) {
        float4 p = pos4[i];
        lo[0] = fminf(lo[0], p.x); lo[1] = fminf(lo[1], p.y); lo[2] = fminf(lo[2], p.z);
        hi[0] = fmaxf(hi[0], p.x); hi[1] = fmaxf(hi[1], p.y); hi[2] = fmaxf(hi[2], p.z);
    }
    __shared__ float slo[3][32], shi[3][32];
#pragma unroll
    for (int d = 0; d < 3; ++d) {
        for (int o = 16; o > 0; o >>= 1) {
            lo[d] = fminf(lo[d], __shfl_xor_sync(0xffffffffu, lo[d], o));
            hi[d] = fmaxf(hi[d], __shfl_xor_sync(0xffffffffu, hi[d], o));
        }
    }
    int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0)
        for (int d = 0; d < 3; ++d) { slo[d][wid] = lo[d]; shi[d][wid] = hi[d]; }
    __syncthreads();
    if (threadIdx.x == 0) {
        int nw = blockDim.x >> 5;
        int g[3];
        GridGeom gm;
        for (int d = 0; d < 3; ++d) {
            float l = 3.4e38f, h = -3.4e38f;
            for (int w = 0; w < nw; ++w) { l = fminf(l, slo[d][w]); h = fmaxf(h, shi[d][w]); }
            if (!(h >= l)) { l = 0.f; h = 0.f; }   // empty replica or non-finite
            const double ext = (double)h - (double)l;   // exact for float inputs
            const int gd = cells_across(ext, gp.rl, gp.gmax);
            g[d] = gd;
            gm.org[d] = (double)l;
            gm.inv[d] = ext > 0.0 ? (double)gd / ext : 0.0;
        }
        dims[r] = make_int4(g[0], g[1], g[2], r * gp.cells_per_rep);
        geom[r] = gm;
    }
}

// Cell coordinate of x along one dimension: floor((x - o) inv) in float64
// (periodic: wrapped into [0, g); open: clamped, only rounding can leave the range).
__device__ __forceinline__ int cell_coord(float x, double o, double iv, int g, int periodic)
{
    const double u = floor(((double)x - o) * iv);
    if (periodic) {
        if (!(fabs(u) < 1.0e15)) return 0;   // non-finite or absurd positions (flagged elsewhere)
        double w = u - (double)g * floor(u / (double)g);
        int c = (int)w;
        return c < 0 ? 0 : (c >= g ? g - 1 : c);
    }
    if (!(u >= 0.0)) return 0;               // also NaN
    return u >= (double)g ? g - 1 : (int)u;
}

__global__ void k_cell_assign(int n, const float4* __restrict__ pos4, const int32_t* __restrict__ atom_rep,
                              const int4* __restrict__ dims, const GridGeom* __restrict__ geom, int periodic,
                              int32_t* __restrict__ cell_of, int32_t* __restrict__ cell_cnt)
{
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    int r = atom_rep[i];
    float4 p = pos4[i];
    int4 g = dims[r];
    const GridGeom gm = geom[r];
    int cx = cell_coord(p.x, gm.org[0], gm.inv[0], g.x, periodic);
    int cy = cell_coord(p.y, gm.org[1], gm.inv[1], g.y, periodic);
    int cz = cell_coord(p.z, gm.org[2], gm.inv[2], g.z, periodic);
    int cell = g.w + cx + g.x * (cy + g.y * cz);
    cell_of[i] = cell;
    atomicAdd(&cell_cnt[cell], 1);
}

__global__ void k_cell_fill(int n, const int32_t* __restrict__ cell_of, const int32_t* __restrict__ cell_start,
                            int32_t* __restrict__ cell_fill, int32_t* __restrict__ cell_atoms)
{
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    int cell = cell_of[i];
    int slot = atomicAdd(&cell_fill[cell], 1);
    cell_atoms[cell_start[cell] + slot] = i;
}

// One warp per cell: the cell's atoms in ascending caller index (the fill above
// places them in arrival order), so the slot order is a function of the
// positions alone.
__global__ void k_cell_order(int ncell, const int32_t* __restrict__ cell_start,
                             const int32_t* __restrict__ cell_atoms, int32_t* __restrict__ perm)
{
    int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int lane = threadIdx.x & 31;
    int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int cell = warp; cell < ncell; cell += nwarps) {
        int a = cell_start[cell], b = cell_start[cell + 1];
        for (int k = a + lane; k < b; k += 32) {
            int v = cell_atoms[k];
            int rank = 0;
            for (int t = a; t < b; ++t) rank += cell_atoms[t] < v;
            perm[a + rank] = v;
        }
    }
}

// slot-order positions and cells from the caller-order ones
__global__ void k_gather_slots(int n, const int32_t* __restrict__ perm, const float4* __restrict__ posc4,
                               const int32_t* __restrict__ cell_of, float4* __restrict__ pos4,
                               int32_t* __restrict__ cell_slot)
{
    int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= n) return;
    const int i = perm[k];
    pos4[k] = posc4[i];
    cell_slot[k] = cell_of[i];
}

// float64 pair test, each operation rounded separately (no contraction)
__device__ __forceinline__ bool pair_in_list(float4 pi, float4 pj, double rl2, const Box& box)
{
    double dx = __dsub_rn((double)pj.x, (double)pi.x);
    double dy = __dsub_rn((double)pj.y, (double)pi.y);
    double dz = __dsub_rn((double)pj.z, (double)pi.z);
    if (box.periodic) {
        double Lx = (double)box.L[0], Ly = (double)box.L[1], Lz = (double)box.L[2];
        dx = __dsub_rn(dx, __dmul_rn(Lx, rint(__ddiv_rn(dx, Lx))));
        dy = __dsub_rn(dy, __dmul_rn(Ly, rint(__ddiv_rn(dy, Ly))));
        dz = __dsub_rn(dz, __dmul_rn(Lz, rint(__ddiv_rn(dz, Lz))));
    }
    double d2 = __dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy));
    d2 = __dadd_rn(d2, __dmul_rn(dz, dz));
    return d2 < rl2;
}

// Visit every candidate j (cells around atom i's cell) passing the list test.
// With cell_atoms == nullptr the atoms are already in cell order: the
// candidates of a cell are the index range cell_start[cell] .. cell_start[cell+1].
template <class Fn>
__device__ __forceinline__ void for_each_neighbor(int i, const float4* __restrict__ pos4,
                                                  const int32_t* __restrict__ atom_rep,
                                                  const int32_t* __restrict__ cell_of,
                                                  const int4* __restrict__ dims,
                                                  const int32_t* __restrict__ cell_start,
                                                  const int32_t* __restrict__ cell_atoms, double rl2,
                                                  const Box& box, Fn&& fn)
{
    int r = atom_rep[i];
    int4 g = dims[r];
    int local = cell_of[i] - g.w;
    int cx = local % g.x, cy = (local / g.x) % g.y, cz = local / (g.x * g.y);
    float4 pi = pos4[i];
    // Stencil per dimension: the cell and its two neighbours (wrapped when
    // periodic, cut at the grid's edge when not).  A periodic dimension with
    // fewer than 3 cells has every cell within reach: it visits each cell once
    // by absolute index (wrapped offsets would visit one cell twice).
    const bool allx = box.periodic && g.x < 3, ally = box.periodic && g.y < 3, allz = box.periodic && g.z < 3;
    const int lox = allx ? 0 : -1, hix = allx ? g.x - 1 : 1;
    const int loy = ally ? 0 : -1, hiy = ally ? g.y - 1 : 1;
    const int loz = allz ? 0 : -1, hiz = allz ? g.z - 1 : 1;
    for (int oz = loz; oz <= hiz; ++oz) {
        int z = allz ? oz : cz + oz;
        if (box.periodic) { if (!allz) z = (z + g.z) % g.z; }
        else if (z < 0 || z >= g.z) continue;
        for (int oy = loy; oy <= hiy; ++oy) {
            int y = ally ? oy : cy + oy;
            if (box.periodic) { if (!ally) y = (y + g.y) % g.y; }
            else if (y < 0 || y >= g.y) continue;
            for (int ox = lox; ox <= hix; ++ox) {
                int x = allx ? ox : cx + ox;
                if (box.periodic) { if (!allx) x = (x + g.x) % g.x; }
                else if (x < 0 || x >= g.x) continue;
                int cell = g.w + x + g.x * (y + g.y * z);
                int a = cell_start[cell], b = cell_start[cell + 1];
                for (int k = a; k < b; ++k) {
                    int j = cell_atoms ? cell_atoms[k] : k;
                    if (j == i) continue;
                    if (pair_in_list(pi, pos4[j], rl2, box)) fn(j);
                }
            }
        }
    }
}

__global__ void k_count(int n, const float4* __restrict__ pos4, const int32_t* __restrict__ atom_rep,
                        const int32_t* __restrict__ cell_of, const int4* __restrict__ dims,
                        const int32_t* __restrict__ cell_start, const int32_t* __restrict__ cell_atoms,
                        double rl2, const Box box, int32_t* __restrict__ rowcnt)
{
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    int cnt = 0;
    for_each_neighbor(i, pos4, atom_rep, cell_of, dims, cell_start, cell_atoms, rl2, box, [&](int) { ++cnt; });
    rowcnt[i] = cnt;
}

__global__ void k_fill(int n, const float4* __restrict__ pos4, const int32_t* __restrict__ atom_rep,
                       const int32_t* __restrict__ cell_of, const int4* __restrict__ dims,
                       const int32_t* __restrict__ cell_start, const int32_t* __restrict__ cell_atoms, double rl2,
                       const Box box, const int32_t* __restrict__ row_ptr, long long cap, DevMeta* meta,
                       int32_t* __restrict__ coltmp, int32_t* __restrict__ erow)
{
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    if (meta->n_edges > cap) return;
    int e = row_ptr[i];
    for_each_neighbor(i, pos4, atom_rep, cell_of, dims, cell_start, cell_atoms, rl2, box, [&](int j) {
        coltmp[e] = j;
        erow[e] = i;
        ++e;
    });
}

// one warp per row: stable placement by rank (entries of a row are distinct)
__global__ void k_sort_rows(int n, const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ coltmp,
                            long long cap, const DevMeta* meta, int32_t* __restrict__ col)
{
    if (meta->n_edges > cap) return;
    int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int lane = threadIdx.x & 31;
    int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int i = warp; i < n; i += nwarps) {
        int a = row_ptr[i], b = row_ptr[i + 1];
        for (int k = a + lane; k < b; k += 32) {
            int v = coltmp[k];
            int rank = 0;
            for (int t = a; t < b; ++t) rank += coltmp[t] < v;
            col[a + rank] = v;
        }
    }
}

// rev[e] = position of the reverse edge (binary search of i in row j)
__global__ void k_rev(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                      const int32_t* __restrict__ erow, long long cap, const DevMeta* meta,
                      int32_t* __restrict__ rev)
{
    long long E = meta->n_edges;
    if (E > cap) return;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < E;
         e += (long long)gridDim.x * blockDim.x) {
        int i = erow[e], j = col[e];
        int lo = row_ptr[j], hi = row_ptr[j + 1] - 1, found = -1;
        while (lo <= hi) {
            int mid = (lo + hi) >> 1;
            int v = col[mid];
            if (v == i) { found = mid; break; }
            if (v < i) lo = mid + 1; else hi = mid - 1;
        }
        rev[e] = found;
    }
}

// erow must describe the sorted list too: rows are unchanged by sorting
// within a row, so the unsorted erow is already correct.

// Row partition of the tensor-core kernels: CTA c takes whole rows holding
// about one share of the edges (at least a few tiles).  row_ptr is the exclusive
// prefix sum over the rows of the edges to balance, row_ptr[n] their total.
__global__ void k_partition(int n, int ncta, const int32_t* __restrict__ row_ptr, long long cap,
                            const DevMeta* meta, int32_t* __restrict__ part)
{
    int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c > ncta) return;
    const long long E = meta->n_edges > cap ? 0 : row_ptr[n];
    long long share = (E + ncta - 1) / ncta;
    if (share < 2 * TILE_E) share = 2 * TILE_E;
    share = (share + TILE_E - 1) / TILE_E * TILE_E;
    if (c == 0) { part[0] = 0; return; }
    if (c == ncta) { part[c] = n; return; }
    long long target = (long long)c * share;
    if (target >= E) { part[c] = n; return; }
    // first row whose start is >= target
    int lo = 0, hi = n;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if ((long long)row_ptr[mid] < target) lo = mid + 1; else hi = mid;
    }
    part[c] = lo;
}

// Per row, the edges the tensor-core kernels will carry at the build's positions:
// those inside the cutoff (cnt), and of them those that own their pair (cnt_half,
// the half list that visits each unordered pair once) and the others (cnt_rev, its
// complement).  The distance is the masking pass's own expression, so the counts
// equal what it keeps at these positions; the row partitions balance them.  One
// warp per row.
__global__ void k_cut_counts(int n, const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                             const float4* __restrict__ pos4, const Box box, float rc, long long cap,
                             const DevMeta* meta, int32_t* __restrict__ cnt, int32_t* __restrict__ cnt_half,
                             int32_t* __restrict__ cnt_rev)
{
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const bool over = meta->n_edges > cap;
    for (int i = warp; i < n; i += nwarps) {
        int c = 0, ch = 0;
        if (!over) {
            const float4 pi = pos4[i];
            for (int e = row_ptr[i] + lane; e < row_ptr[i + 1]; e += 32) {
                const int j = col[e];
                float3 v;
                const float d = edge_distance(pi, pos4[j], box, v);
                if (d < rc && d > 0.f) {
                    ++c;
                    ch += owns_pair(i, j);
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            c += __shfl_xor_sync(0xffffffffu, c, o);
            ch += __shfl_xor_sync(0xffffffffu, ch, o);
        }
        if (lane == 0) {
            cnt[i] = c;
            cnt_half[i] = ch;
            cnt_rev[i] = c - ch;
        }
    }
}

__global__ void k_check_capacity(long long cap, DevMeta* meta)
{
    if (meta->n_edges > cap) set_flag(meta, SCHNET_FLAG_CAPACITY);
}

// Build from the caller-order positions d_pos: cell grid and cell sort in the
// caller's order, then the slot permutation, then the list itself in slot order.
cudaError_t launch_build_neighbors(schnet_ctx* c, const float* d_pos)
{
    Workspace& w = c->ws;
    const int N = c->N, R = c->R;
    GridParams gp;
    gp.periodic = c->cfg.periodic;
    gp.gp[0] = c->gdim[0]; gp.gp[1] = c->gdim[1]; gp.gp[2] = c->gdim[2];
    gp.rl = (double)c->cfg.cutoff + (double)c->cfg.skin;
    gp.gmax = GMAX_NONPERIODIC;
    gp.cells_per_rep = c->ncell / R;
    cudaError_t err;
    const int nb = (N + 255) / 256;
    float4* posc4 = w.ref4;   // caller-order positions; replaced by the slot-order reference at the end

    k_pack_positions<<<nb, 256, 0, c->s>>>(N, d_pos, nullptr, posc4, nullptr, 0, 0.f, w.meta);
    k_replica_grid<<<R, 256, 0, c->s>>>(R, w.rep_off, posc4, gp, c->box, w.rgrid_dims, w.rgrid_geom);
    cudaMemsetAsync(w.cell_cnt, 0, sizeof(int32_t) * (c->ncell + 1), c->s);
    cudaMemsetAsync(w.cell_fill, 0, sizeof(int32_t) * (c->ncell + 1), c->s);
    k_cell_assign<<<nb, 256, 0, c->s>>>(N, posc4, w.atom_rep, w.rgrid_dims, w.rgrid_geom, gp.periodic,
                                        w.cell_of, w.cell_cnt);
    c->launches += 3;
    if ((err = scan_exclusive(c, w.cell_cnt, c->ncell, w.cell_start, nullptr)) != cudaSuccess) return err;
    k_cell_fill<<<nb, 256, 0, c->s>>>(N, w.cell_of, w.cell_start, w.cell_fill, w.cell_atoms);
    k_cell_order<<<c->nsm * 8, 256, 0, c->s>>>(c->ncell, w.cell_start, w.cell_atoms, w.perm);
    k_gather_slots<<<nb, 256, 0, c->s>>>(N, w.perm, posc4, w.cell_of, w.pos4, w.cell_slot);
    // slot space from here on: a replica's slots are its caller index range, so atom_rep serves both
    const int nb128 = (N + 127) / 128;
    k_count<<<nb128, 128, 0, c->s>>>(N, w.pos4, w.atom_rep, w.cell_slot, w.rgrid_dims, w.cell_start, nullptr,
                                     c->rl2, c->box, w.rowcnt);
    c->launches += 4;
    if ((err = scan_exclusive(c, w.rowcnt, N, w.row_ptr, &w.meta->n_edges)) != cudaSuccess) return err;
    k_check_capacity<<<1, 1, 0, c->s>>>(c->cap, w.meta);
    k_fill<<<nb128, 128, 0, c->s>>>(N, w.pos4, w.atom_rep, w.cell_slot, w.rgrid_dims, w.cell_start, nullptr,
                                    c->rl2, c->box, w.row_ptr, c->cap, w.meta, w.coltmp, w.erow);
    int nsort = c->nsm * 8;
    k_sort_rows<<<nsort, 256, 0, c->s>>>(N, w.row_ptr, w.coltmp, c->cap, w.meta, w.col);
    k_rev<<<c->nsm * 8, 256, 0, c->s>>>(w.row_ptr, w.col, w.erow, c->cap, w.meta, w.rev);
    // the row partitions of the full and the half list, balanced on the edges inside the
    // cutoff at the build's positions (rowcnt is free scratch once the list is built)
    k_cut_counts<<<c->nsm * 8, 256, 0, c->s>>>(N, w.row_ptr, w.col, w.pos4, c->box, c->cfg.cutoff, c->cap, w.meta,
                                               w.rowcnt, w.hcnt, w.rcnt);
    c->launches += 5;
    if ((err = scan_exclusive(c, w.rowcnt, N, w.rowcnt, nullptr)) != cudaSuccess) return err;   // in place
    if ((err = scan_exclusive(c, w.hcnt, N, w.hcnt, nullptr)) != cudaSuccess) return err;
    if ((err = scan_exclusive(c, w.rcnt, N, w.rcnt, nullptr)) != cudaSuccess) return err;
    const int npb = (c->ncta + 1 + 127) / 128;
    k_partition<<<npb, 128, 0, c->s>>>(N, c->ncta, w.rowcnt, c->cap, w.meta, w.part);
    k_partition<<<npb, 128, 0, c->s>>>(N, c->ncta, w.hcnt, c->cap, w.meta, w.part_h);
    k_partition<<<npb, 128, 0, c->s>>>(N, c->ncta, w.rcnt, c->cap, w.meta, w.part_r);
    cudaMemcpyAsync(w.ref4, w.pos4, sizeof(float4) * N, cudaMemcpyDeviceToDevice, c->s);
    c->launches += 3;
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// the list and per-atom values in the caller's atom order (inspection taps)
// ---------------------------------------------------------------------------
__global__ void k_caller_rowlen(int n, const int32_t* __restrict__ perm, const int32_t* __restrict__ row_ptr,
                                int32_t* __restrict__ cnt)
{
    int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= n) return;
    cnt[perm[k]] = row_ptr[k + 1] - row_ptr[k];
}

// one warp per slot row: its columns, as caller indices, at the caller row's place
__global__ void k_caller_cols(int n, const int32_t* __restrict__ perm, const int32_t* __restrict__ row_ptr,
                              const int32_t* __restrict__ col, const int32_t* __restrict__ row_ptr_c, long long cap,
                              const DevMeta* meta, int32_t* __restrict__ col_c)
{
    if (meta->n_edges > cap) return;
    int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int lane = threadIdx.x & 31;
    int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int k = warp; k < n; k += nwarps) {
        const int a = row_ptr[k], b = row_ptr[k + 1], base = row_ptr_c[perm[k]];
        for (int e = a + lane; e < b; e += 32) col_c[base + (e - a)] = perm[col[e]];
    }
}

__global__ void k_scatter_atoms(int n, const int32_t* __restrict__ perm, const float* __restrict__ v,
                                float* __restrict__ out)
{
    int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k < n) out[perm[k]] = v[k];
}

__global__ void k_rev_rows(int n, const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                           long long cap, const DevMeta* meta, int32_t* __restrict__ rev);

// Caller-order CSR of the current list in (row_ptr, col, rev) = (rowcnt, ccol,
// cidx): scratch that only a build (rowcnt, coltmp) or the start of the next
// energy evaluation (ccol, cidx) rewrites.
cudaError_t launch_caller_order_list(schnet_ctx* c, const int32_t** row_ptr, const int32_t** col,
                                     const int32_t** rev)
{
    Workspace& w = c->ws;
    const int N = c->N;
    cudaError_t err;
    k_caller_rowlen<<<(N + 255) / 256, 256, 0, c->s>>>(N, w.perm, w.row_ptr, w.rowcnt);
    c->launches += 1;
    if ((err = scan_exclusive(c, w.rowcnt, N, w.rowcnt, nullptr)) != cudaSuccess) return err;   // in place
    k_caller_cols<<<c->nsm * 8, 256, 0, c->s>>>(N, w.perm, w.row_ptr, w.col, w.rowcnt, c->cap, w.meta, w.coltmp);
    k_sort_rows<<<c->nsm * 8, 256, 0, c->s>>>(N, w.rowcnt, w.coltmp, c->cap, w.meta, w.ccol);
    k_rev_rows<<<c->nsm * 8, 256, 0, c->s>>>(N, w.rowcnt, w.ccol, c->cap, w.meta, w.cidx);
    c->launches += 3;
    *row_ptr = w.rowcnt;
    *col = w.ccol;
    *rev = w.cidx;
    return cudaGetLastError();
}

cudaError_t launch_scatter_atoms(schnet_ctx* c, const float* v, float* out)
{
    k_scatter_atoms<<<(c->N + 255) / 256, 256, 0, c->s>>>(c->N, c->ws.perm, v, out);
    c->launches += 1;
    return cudaGetLastError();
}

}  // namespace schnet

// ===========================================================================
// Allocation-free neighbour build (schnet_build_neighbors_noalloc)
//
// For callers that cannot allocate device memory at the point of the call --
// for example a host application that hands this library only the buffers it
// already owns, or a runtime that forbids allocation while it is running --
// the build's scratch (packed positions, cell grid, cell counts and starts,
// row counts, scan partial sums, status) lives in one fixed-size device array
// defined in this file.  Every device that loads the library keeps that array
// until the process exits.  The caller supplies positions and the output
// buffers; the row-sorted columns are staged in the caller's `rev` buffer
// before the transpose map overwrites it, so no per-edge scratch is needed.
// ===========================================================================
namespace schnet {

constexpr int NA_MAX_ATOMS = 65536;
constexpr int NA_MAX_REPLICAS = 1024;
constexpr int NA_MAX_CELLS = 131072;

// carve offsets (bytes) inside the static array
constexpr size_t na_align(size_t x) { return (x + 255) / 256 * 256; }
constexpr size_t NA_OFF_META = 0;
constexpr size_t NA_OFF_POS4 = na_align(NA_OFF_META + sizeof(DevMeta));
constexpr size_t NA_OFF_AREP = na_align(NA_OFF_POS4 + sizeof(float4) * NA_MAX_ATOMS);
constexpr size_t NA_OFF_CELLOF = na_align(NA_OFF_AREP + sizeof(int32_t) * NA_MAX_ATOMS);
constexpr size_t NA_OFF_CATOMS = na_align(NA_OFF_CELLOF + sizeof(int32_t) * NA_MAX_ATOMS);
constexpr size_t NA_OFF_ROWCNT = na_align(NA_OFF_CATOMS + sizeof(int32_t) * NA_MAX_ATOMS);
constexpr size_t NA_OFF_CCNT = na_align(NA_OFF_ROWCNT + sizeof(int32_t) * (NA_MAX_ATOMS + 1));
constexpr size_t NA_OFF_CSTART = na_align(NA_OFF_CCNT + sizeof(int32_t) * (NA_MAX_CELLS + 1));
constexpr size_t NA_OFF_CFILL = na_align(NA_OFF_CSTART + sizeof(int32_t) * (NA_MAX_CELLS + 1));
constexpr size_t NA_OFF_DIMS = na_align(NA_OFF_CFILL + sizeof(int32_t) * (NA_MAX_CELLS + 1));
constexpr size_t NA_OFF_GEOM = na_align(NA_OFF_DIMS + sizeof(int4) * NA_MAX_REPLICAS);
constexpr size_t NA_OFF_SCAN = na_align(NA_OFF_GEOM + sizeof(GridGeom) * NA_MAX_REPLICAS);
constexpr size_t NA_BYTES = na_align(NA_OFF_SCAN + sizeof(long long) * SCAN_TILE);   // about 3.6 MB

static __device__ __align__(256) unsigned char g_noalloc_scratch[NA_BYTES];

// Per-device address of g_noalloc_scratch, looked up once with the device current.
static void* g_noalloc_ptr[64] = {};
static std::mutex g_noalloc_mu;

static cudaError_t noalloc_scratch(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

// atom -> replica map from the offsets (binary search)
__global__ void k_atom_replica(int n, int R, const int32_t* __restrict__ rep_off, int32_t* __restrict__ atom_rep)
{
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    int lo = 0, hi = R - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (rep_off[mid] <= i) lo = mid; else hi = mid - 1;
    }
    atom_rep[i] = lo;
}

// rev[e] by a warp per row (the row of an edge is known from the loop)
__global__ void k_rev_rows(int n, const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                           long long cap, const DevMeta* meta, int32_t* __restrict__ rev)
{
    if (meta->n_edges > cap) return;
    int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int lane = threadIdx.x & 31;
    int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int i = warp; i < n; i += nwarps) {
        for (int e = row_ptr[i] + lane; e < row_ptr[i + 1]; e += 32) {
            int j = col[e];
            int lo = row_ptr[j], hi = row_ptr[j + 1] - 1, found = -1;
            while (lo <= hi) {
                int mid = (lo + hi) >> 1;
                int v = col[mid];
                if (v == i) { found = mid; break; }
                if (v < i) lo = mid + 1; else hi = mid - 1;
            }
            rev[e] = found;
        }
    }
}

// edge count and status bits (non-finite positions, list over capacity) out to the caller
__global__ void k_copy_edge_count(DevMeta* meta, long long cap, int64_t* out, uint32_t* flags)
{
    if (meta->n_edges > cap) set_flag(meta, SCHNET_FLAG_CAPACITY);
    *out = meta->n_edges;
    if (flags) *flags = meta->status;
}

static cudaError_t scan_exclusive_raw(cudaStream_t s, const int32_t* in, int n, int32_t* out, long long* total64,
                                      long long* tmp)
{
    int ntiles = (n + SCAN_TILE - 1) / SCAN_TILE;
    if (ntiles < 1) ntiles = 1;
    if (ntiles > SCAN_TILE) return cudaErrorInvalidValue;
    k_scan_tiles<<<ntiles, SCAN_BLOCK, 0, s>>>(in, n, tmp);
    k_scan_sums<<<1, SCAN_BLOCK, 0, s>>>(tmp, ntiles);
    k_scan_apply<<<ntiles, SCAN_BLOCK, 0, s>>>(in, n, tmp, out, total64, ntiles);
    return cudaGetLastError();
}

}  // namespace schnet

extern "C" schnet_status schnet_build_neighbors_noalloc(const float* d_pos, int32_t n_atoms, int32_t n_replicas,
                                                        const int32_t* d_replica_offsets, float cutoff, float skin,
                                                        int32_t periodic, const float* box, int32_t* d_row_ptr,
                                                        int32_t* d_col, int32_t* d_rev, int64_t edge_capacity,
                                                        int64_t* d_n_edges, uint32_t* d_flags, void* cuda_stream)
{
    using namespace schnet;
    if (!d_pos || !d_replica_offsets || !d_row_ptr || !d_col || !d_rev || !d_n_edges || n_atoms < 1 ||
        n_replicas < 1 || edge_capacity < 1 || !(cutoff > 0.f) || !(skin >= 0.f) || (periodic && !box))
        return SCHNET_ERR_INVALID_ARG;
    // An error left pending by someone else's earlier launch is theirs to read: report it
    // without clearing it, so that the launch-error check at the end sees only this call's.
    if (cudaPeekAtLastError() != cudaSuccess) return SCHNET_ERR_CUDA;
    const double rl = (double)cutoff + (double)skin;
    int gdim[3] = {GMAX_NONPERIODIC, GMAX_NONPERIODIC, GMAX_NONPERIODIC};
    Box bx;
    bx.periodic = periodic ? 1 : 0;
    for (int d = 0; d < 3; ++d) {
        bx.L[d] = periodic ? box[d] : 0.f;
        bx.invL[d] = periodic ? 1.0f / box[d] : 0.f;
        if (periodic) {
            if (!(box[d] >= 2.0f * (cutoff + skin))) return SCHNET_ERR_UNSUPPORTED;
            gdim[d] = cells_across((double)box[d], rl, GMAX_PERIODIC);
        }
    }
    const long long cells_per_rep = (long long)gdim[0] * gdim[1] * gdim[2];
    const long long ncell = cells_per_rep * n_replicas;
    if (n_atoms > NA_MAX_ATOMS || n_replicas > NA_MAX_REPLICAS || ncell > NA_MAX_CELLS ||
        edge_capacity > 0x7fffffffLL)
        return SCHNET_ERR_UNSUPPORTED;

    uint8_t* base = nullptr;
    if (noalloc_scratch(reinterpret_cast<void**>(&base)) != cudaSuccess) return SCHNET_ERR_CUDA;
    DevMeta* meta = reinterpret_cast<DevMeta*>(base + NA_OFF_META);
    float4* pos4 = reinterpret_cast<float4*>(base + NA_OFF_POS4);
    int32_t* arep = reinterpret_cast<int32_t*>(base + NA_OFF_AREP);
    int32_t* cell_of = reinterpret_cast<int32_t*>(base + NA_OFF_CELLOF);
    int32_t* catoms = reinterpret_cast<int32_t*>(base + NA_OFF_CATOMS);
    int32_t* rowcnt = reinterpret_cast<int32_t*>(base + NA_OFF_ROWCNT);
    int32_t* ccnt = reinterpret_cast<int32_t*>(base + NA_OFF_CCNT);
    int32_t* cstart = reinterpret_cast<int32_t*>(base + NA_OFF_CSTART);
    int32_t* cfill = reinterpret_cast<int32_t*>(base + NA_OFF_CFILL);
    int4* dims = reinterpret_cast<int4*>(base + NA_OFF_DIMS);
    GridGeom* geom = reinterpret_cast<GridGeom*>(base + NA_OFF_GEOM);
    long long* scan_tmp = reinterpret_cast<long long*>(base + NA_OFF_SCAN);

    cudaStream_t s = (cudaStream_t)cuda_stream;
    const int N = n_atoms, R = n_replicas;
    const int nb = (N + 255) / 256, nb128 = (N + 127) / 128;
    GridParams gp;
    gp.periodic = bx.periodic;
    gp.gp[0] = gdim[0]; gp.gp[1] = gdim[1]; gp.gp[2] = gdim[2];
    gp.rl = rl;
    gp.gmax = GMAX_NONPERIODIC;
    gp.cells_per_rep = (int)cells_per_rep;
    const double rl2 = rl * rl;
    // scratch that must start at zero: status and edge count, cell counts and fill cursors
    if (cudaMemsetAsync(meta, 0, sizeof(DevMeta), s) != cudaSuccess) return SCHNET_ERR_CUDA;
    if (cudaMemsetAsync(ccnt, 0, sizeof(int32_t) * (ncell + 1), s) != cudaSuccess) return SCHNET_ERR_CUDA;
    if (cudaMemsetAsync(cfill, 0, sizeof(int32_t) * (ncell + 1), s) != cudaSuccess) return SCHNET_ERR_CUDA;
    k_pack_positions<<<nb, 256, 0, s>>>(N, d_pos, nullptr, pos4, nullptr, 0, 0.f, meta);
    k_atom_replica<<<nb, 256, 0, s>>>(N, R, d_replica_offsets, arep);
    k_replica_grid<<<R, 256, 0, s>>>(R, d_replica_offsets, pos4, gp, bx, dims, geom);
    k_cell_assign<<<nb, 256, 0, s>>>(N, pos4, arep, dims, geom, gp.periodic, cell_of, ccnt);
    if (scan_exclusive_raw(s, ccnt, (int)ncell, cstart, nullptr, scan_tmp) != cudaSuccess) return SCHNET_ERR_CUDA;
    k_cell_fill<<<nb, 256, 0, s>>>(N, cell_of, cstart, cfill, catoms);
    k_count<<<nb128, 128, 0, s>>>(N, pos4, arep, cell_of, dims, cstart, catoms, rl2, bx, rowcnt);
    if (scan_exclusive_raw(s, rowcnt, N, d_row_ptr, &meta->n_edges, scan_tmp) != cudaSuccess)
        return SCHNET_ERR_CUDA;
    // unsorted columns staged in the caller's rev buffer; col doubles as the edge-row scratch
    k_fill<<<nb128, 128, 0, s>>>(N, pos4, arep, cell_of, dims, cstart, catoms, rl2, bx, d_row_ptr, edge_capacity,
                                 meta, d_rev, d_col);
    k_sort_rows<<<256, 256, 0, s>>>(N, d_row_ptr, d_rev, edge_capacity, meta, d_col);
    k_rev_rows<<<256, 256, 0, s>>>(N, d_row_ptr, d_col, edge_capacity, meta, d_rev);
    k_copy_edge_count<<<1, 1, 0, s>>>(meta, edge_capacity, d_n_edges, d_flags);
    return cudaGetLastError() == cudaSuccess ? SCHNET_OK : SCHNET_ERR_CUDA;
}
