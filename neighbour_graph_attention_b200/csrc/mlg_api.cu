// mlg_api.cu -- the C ABI of libmlg.so: argument checks, workspace layout and
// kernel launches on the caller's stream.  No allocation, no synchronisation.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "mlg.h"
#include "mlg_common.cuh"
#include "mlg_build.cuh"
#include "mlg_attn.cuh"
#include "mlg_attn_tile.cuh"
#include "mlg_attn_hg.cuh"
#include "mlg_attn_dmma.cuh"
#include "mlg_attn_tc.cuh"
#include "mlg_attn_tc2.cuh"
#include "mlg_attn_tc6.cuh"
#include "mlg_attn_tc7.cuh"
#include "mlg_attn_hgtc.cuh"
#include "mlg_local.cuh"
#include "mlg_verlet.cuh"

using namespace mlg;

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxNnei = 256;
constexpr int kMaxReach = 62;  // stencil reach limit (image packing of the sort key)

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Layout of the build workspace.
struct BuildLayout {
  size_t grid, bbox, cell_count, cell_start, atom_cell, atom_rank, atom_w, recs, pos4, kept, raw,
      partial, sync, total;
  size_t stash, stash_n, total_stash;  // the count-to-fill key stash after `total`
};

int64_t scan_tiles(int64_t n) { return (n + kScanTile - 1) / kScanTile; }

BuildLayout build_layout(int64_t n, int ncell_cap) {
  BuildLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes);
    return o;
  };
  L.grid = take(sizeof(CellGrid));
  L.bbox = take(6 * sizeof(unsigned long long));
  L.cell_count = take((size_t)(ncell_cap + 1) * sizeof(int));
  L.cell_start = take((size_t)(ncell_cap + 1) * sizeof(int));
  L.atom_cell = take((size_t)n * sizeof(int));
  L.atom_rank = take((size_t)n * sizeof(int));
  L.atom_w = take((size_t)n * sizeof(int));
  L.recs = take((size_t)n * sizeof(Rec));
  L.pos4 = take((size_t)n * sizeof(float4));
  L.kept = take((size_t)n * sizeof(int));
  L.raw = take((size_t)n * sizeof(int));
  int64_t tiles = scan_tiles(n > ncell_cap ? n : ncell_cap + 1);
  L.partial = take((size_t)(tiles + 2) * sizeof(long long));
  L.sync = take(sizeof(FusedSync));
  L.total = off;
  L.stash = take((size_t)n * kStashSlots * sizeof(unsigned long long));
  L.stash_n = take((size_t)n * sizeof(int));
  L.total_stash = off;
  return L;
}

bool finite_box(const double* box) {
  for (int k = 0; k < 9; ++k)
    if (!std::isfinite(box[k])) return false;
  return true;
}

// Cell grid that the host can fix: cells along periodic axes (size >= rcut
// plus a margin, so one layer of neighbouring cells covers rcut), caps along
// open axes, the stencil reach, and the total cell budget.
int make_plan(int64_t n, double rcut, const double* box, const uint8_t* pbc, BuildPlan* p) {
  if (n < 1 || n > (int64_t)INT32_MAX / 2 || !(rcut > 0.0) || !std::isfinite(rcut) ||
      box == nullptr || pbc == nullptr || !finite_box(box))
    return MLG_ERR_INVALID_ARG;
  std::memset(p, 0, sizeof(*p));
  const double delta = 1e-6 * (rcut > 1.0 ? rcut : 1.0);
  p->rcd = rcut + delta;
  p->rc2 = rcut * rcut;
  const double budget = (double)(n > 32 ? 2 * n : 64);
  double prod = 1.0;
  int n_open = 0;
  for (int k = 0; k < 3; ++k) {
    p->periodic[k] = pbc[k] ? 1 : 0;
    if (!p->periodic[k]) {
      ++n_open;
      continue;
    }
    for (int c = 0; c < 3; ++c)
      if (c != k && box[3 * k + c] != 0.0) return MLG_ERR_UNSUPPORTED;  // sheared cell
    double L = box[3 * k + k];
    if (!(L > 0.0)) return MLG_ERR_INVALID_ARG;
    p->L[k] = L;
    p->invL[k] = 1.0 / L;
    double q = std::floor(L / p->rcd);
    p->n_fixed[k] = q < 1.0 ? 1 : (q > 1024.0 ? 1024 : (int)q);
    prod *= p->n_fixed[k];
  }
  // coarsen periodic axes until the grid fits the cell budget
  while (prod > budget) {
    int kmax = -1;
    for (int k = 0; k < 3; ++k)
      if (p->periodic[k] && (kmax < 0 || p->n_fixed[k] > p->n_fixed[kmax])) kmax = k;
    if (kmax < 0 || p->n_fixed[kmax] == 1) break;
    prod /= p->n_fixed[kmax];
    p->n_fixed[kmax] = (p->n_fixed[kmax] + 1) / 2;
    prod *= p->n_fixed[kmax];
  }
  for (int k = 0; k < 3; ++k) {
    if (!p->periodic[k]) continue;
    p->inv_h[k] = (double)p->n_fixed[k] / p->L[k];
    double reach = std::ceil(p->rcd * (double)p->n_fixed[k] / p->L[k]);
    if (reach > kMaxReach) return MLG_ERR_UNSUPPORTED;  // box far smaller than rcut
    p->D_fixed[k] = reach < 1.0 ? 1 : (int)reach;
    if (p->D_fixed[k] > p->max_reach) p->max_reach = p->D_fixed[k];
  }
  int open_cap = 1;
  if (n_open > 0) {
    double room = budget / prod;
    open_cap = (int)std::floor(std::pow(room, 1.0 / n_open) + 1e-9);
    if (open_cap < 1) open_cap = 1;
    if (open_cap > 1024) open_cap = 1024;
  }
  double cells = prod;
  for (int k = 0; k < 3; ++k)
    if (!p->periodic[k]) {
      p->n_open_max[k] = open_cap;
      cells *= open_cap;
    }
  p->any_open = n_open > 0;
  p->ncell_cap = (int)cells;
  return MLG_OK;
}

void taylor_coeffs(double* c) {
  // (-1)^k / (2k+1)!, by c_k = -c_{k-1} / ((2k)(2k+1)), each division rounded
  c[0] = 1.0;
  for (int k = 1; k < 12; ++k) c[k] = -c[k - 1] / (double)((2 * k) * (2 * k + 1));
}

// Host-side caches.  A kernel's attributes and occupancy, and a device's SM
// count, do not change while the process runs, so the queries and attribute
// settings behind a launch happen once per kernel and device rather than on
// every call (they cost microseconds of host time each).
struct KernelCacheEntry {
  const void* fn;
  int dev;
  size_t smem_set;  // largest dynamic shared memory size set so far (0: none)
  int nt;           // occupancy query: threads, shared memory, result
  size_t smem_occ;
  int blocks;
};
std::mutex g_kc_mu;
constexpr int kKernelCacheMax = 512;
KernelCacheEntry g_kc[kKernelCacheMax];
int g_kc_n = 0;

int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}

// Entry for (fn, dev), created if absent (nullptr when the cache is full).
KernelCacheEntry* kernel_cache(const void* fn, int dev) {
  for (int i = 0; i < g_kc_n; ++i)
    if (g_kc[i].fn == fn && g_kc[i].dev == dev) return &g_kc[i];
  if (g_kc_n == kKernelCacheMax) return nullptr;
  g_kc[g_kc_n] = KernelCacheEntry{fn, dev, 0, 0, 0, 0};
  return &g_kc[g_kc_n++];
}

// Blocks of `kern` that fit on one SM by registers, shared memory, warps.
template <typename K>
int resident_blocks_uncached(K kern, int nt, size_t dyn_smem) {
  cudaFuncAttributes fa;
  int dev = 0, regs_sm = 65536, smem_sm = 233472, reserved = 1024, thr_sm = 2048;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
  cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  cudaDeviceGetAttribute(&thr_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev);
  const int regs_warp = ((fa.numRegs * 32 + 255) / 256) * 256;
  int by_regs = regs_sm / (regs_warp * (nt / 32));
  int by_smem = (int)(smem_sm / (dyn_smem + fa.sharedSizeBytes + reserved));
  int by_thr = thr_sm / nt;
  int b = by_regs < by_smem ? by_regs : by_smem;
  b = b < by_thr ? b : by_thr;
  return b < 1 ? 1 : b;
}

template <typename K>
int resident_blocks(K kern, int nt, size_t dyn_smem) {
  const void* fn = reinterpret_cast<const void*>(kern);
  const int dev = current_device();
  {
    std::lock_guard<std::mutex> lk(g_kc_mu);
    KernelCacheEntry* e = kernel_cache(fn, dev);
    if (e != nullptr && e->blocks > 0 && e->nt == nt && e->smem_occ == dyn_smem) return e->blocks;
  }
  const int b = resident_blocks_uncached(kern, nt, dyn_smem);
  std::lock_guard<std::mutex> lk(g_kc_mu);
  if (KernelCacheEntry* e = kernel_cache(fn, dev)) {
    e->nt = nt;
    e->smem_occ = dyn_smem;
    e->blocks = b;
  }
  return b;
}

// Allow `smem` bytes of dynamic shared memory and ask for the largest
// carveout, so that the occupancy the shared memory allows is the occupancy
// the launch gets.
template <typename K>
void prefer_shared(K kern, size_t smem) {
  const void* fn = reinterpret_cast<const void*>(kern);
  const int dev = current_device();
  {
    std::lock_guard<std::mutex> lk(g_kc_mu);
    KernelCacheEntry* e = kernel_cache(fn, dev);
    if (e != nullptr && e->smem_set >= smem && e->smem_set > 0) return;
  }
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                       (int)cudaSharedmemCarveoutMaxShared);
  std::lock_guard<std::mutex> lk(g_kc_mu);
  if (KernelCacheEntry* e = kernel_cache(fn, dev)) e->smem_set = smem > e->smem_set ? smem : e->smem_set;
}

int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MLG_OK : MLG_ERR_CUDA;
}

// Exclusive scan of n ints into TOut offsets [n + 1].
template <typename TOut>
void launch_scan(const int* in, int64_t n, TOut* out, long long* partial, ScanTail tail,
                 cudaStream_t s) {
  if (n <= kScanSingleMax) {
    k_scan_single<TOut><<<1, 1024, 0, s>>>(in, n, out, tail);
    return;
  }
  int tiles = (int)scan_tiles(n);
  k_scan_reduce<<<tiles, kScanThreads, 0, s>>>(in, n, partial, tail.gate);
  k_scan_top<<<1, 1024, 0, s>>>(partial, tiles, tail.gate);
  k_scan_down<TOut><<<tiles, kScanThreads, 0, s>>>(in, n, partial, tiles, out, tail);
}

int check_csr(const mlg_csr* csr) {
  if (csr == nullptr || csr->capacity < 0) return csr ? MLG_ERR_CAPACITY : MLG_ERR_INVALID_ARG;
  if (!csr->row_ptr || !csr->n_edges || !csr->n_truncated || !csr->status)
    return MLG_ERR_INVALID_ARG;
  if (csr->capacity > 0 &&
      (!csr->src || !csr->shift || !csr->vec || !csr->dist || !csr->sw))
    return MLG_ERR_INVALID_ARG;
  return MLG_OK;
}

int sm_count();

// Small systems on per-cell scans take the one-launch build.
bool use_fused_build(const BuildPlan& plan, int64_t n) {
  return plan.max_reach <= 1 && n >= 1 && n <= kFusedMaxAtoms &&
         fused_build_fits<kCellCand>(n, plan.ncell_cap);
}

// Arguments of the build kernels for one system whose workspace starts at w
// (layout L).  The caller adjusts the pointers and offsets of a batch.
BuildArgs make_build_args(const mlg_system* sys, double rcut, double r_on, int32_t nnei_max,
                          const mlg_csr* csr, char* w, const BuildLayout& L) {
  BuildArgs a;
  std::memset(&a, 0, sizeof(a));
  a.n = sys->n_atoms;
  a.coords = sys->coords;
  a.types = sys->types;
  a.n_types = sys->n_types;
  std::memcpy(a.box, sys->box, sizeof(a.box));
  a.rcut = rcut;
  a.r_on = r_on;
  a.rc2 = rcut * rcut;
  a.nnei_max = nnei_max;
  taylor_coeffs(a.taylor);
  a.capacity = csr->capacity;
  a.row_ptr = csr->row_ptr;
  a.src = csr->src;
  a.shift = csr->shift;
  a.vec = csr->vec;
  a.dist = csr->dist;
  a.sw = csr->sw;
  a.n_edges = csr->n_edges;
  a.n_truncated = csr->n_truncated;
  a.status = csr->status;
  a.src_offset = 0;
  a.zero_globals = 1;
  a.grid = reinterpret_cast<CellGrid*>(w + L.grid);
  a.bbox = reinterpret_cast<unsigned long long*>(w + L.bbox);
  a.cell_count = reinterpret_cast<int*>(w + L.cell_count);
  a.cell_start = reinterpret_cast<int*>(w + L.cell_start);
  a.atom_cell = reinterpret_cast<int*>(w + L.atom_cell);
  a.atom_rank = reinterpret_cast<int*>(w + L.atom_rank);
  a.atom_w = reinterpret_cast<int*>(w + L.atom_w);
  a.recs = reinterpret_cast<Rec*>(w + L.recs);
  a.pos4 = reinterpret_cast<float4*>(w + L.pos4);
  a.kept = reinterpret_cast<int*>(w + L.kept);
  a.raw = reinterpret_cast<int*>(w + L.raw);
  a.partial = reinterpret_cast<long long*>(w + L.partial);
  a.stash = nullptr;
  a.stash_n = nullptr;
  a.stash_q = 0;
  return a;
}

// A grid of few cells splits each cell's centres over several CTAs.
int build_nsplit(const BuildPlan& plan) {
  int nsplit = (4 * sm_count() + plan.ncell_cap - 1) / plan.ncell_cap;
  return nsplit < 1 ? 1 : (nsplit > 8 ? 8 : nsplit);
}

// Host checks shared by the single and the batched build.
int check_build_args(double rcut, double r_on, int32_t nnei_max, const mlg_csr* csr) {
  if (!(r_on >= 0.0) || !(r_on < rcut) || !std::isfinite(r_on)) return MLG_ERR_INVALID_ARG;
  if (nnei_max < 1) return MLG_ERR_INVALID_ARG;
  if (nnei_max > kMaxNnei) return MLG_ERR_UNSUPPORTED;
  return check_csr(csr);
}

// The launch chain up to the kept counts: init, [bbox], bin, cell scan,
// scatter, count.  Per-cell scans when every stencil reach is 1 (at most 27
// stencil cells); otherwise (boxes narrower than the cutoff) the per-centre
// scans.
void launch_count_phase(const BuildArgs& a, const BuildPlan& plan, int nsplit,
                        cudaStream_t stream) {
  const int tb = 256;
  const int atom_blocks = (int)((a.n + tb - 1) / tb);
  int init_blocks = (plan.ncell_cap + 1 + tb - 1) / tb;
  if (init_blocks > 1024) init_blocks = 1024;
  k_init<<<init_blocks, tb, 0, stream>>>(a, plan.ncell_cap);
  if (plan.any_open) {
    int bb = atom_blocks < 592 ? atom_blocks : 592;
    k_bbox<<<bb, tb, 0, stream>>>(a, plan);
  }
  k_bin<<<atom_blocks, tb, 0, stream>>>(a, plan);
  launch_scan<int>(a.cell_count, plan.ncell_cap, a.cell_start, a.partial,
                   ScanTail{nullptr, nullptr, 0, a.gate}, stream);
  k_scatter<<<atom_blocks, tb, 0, stream>>>(a);
  if (plan.max_reach <= 1 && a.stash != nullptr) {
    // the count keeps each whole row's keys in the workspace stash
    const size_t sm_count_ = cellscan_smem(false);
    prefer_shared(k_cellscan<false, true>, sm_count_);
    k_cellscan<false, true><<<dim3((unsigned)plan.ncell_cap, (unsigned)nsplit), kScanWarps * 32,
                              sm_count_, stream>>>(a);
  } else if (plan.max_reach <= 1) {
    const size_t sm_count_ = cellscan_smem(false);
    prefer_shared(k_cellscan<false>, sm_count_);
    k_cellscan<false><<<dim3((unsigned)plan.ncell_cap, (unsigned)nsplit), kScanWarps * 32,
                        sm_count_, stream>>>(a);
  } else {
    k_count<<<(int)((a.n + kCountWarps - 1) / kCountWarps), kCountWarps * 32, 0, stream>>>(a);
  }
}

// The fill, once row_ptr holds the row starts.
void launch_fill_phase(const BuildArgs& a, const BuildPlan& plan, int nsplit,
                       cudaStream_t stream) {
  if (plan.max_reach <= 1 && a.stash != nullptr) {
    const size_t sm_fill = cellscan_smem(true);
    prefer_shared(k_cellscan<true, true>, sm_fill);
    k_cellscan<true, true><<<dim3((unsigned)plan.ncell_cap, (unsigned)nsplit), kScanWarps * 32,
                             sm_fill, stream>>>(a);
  } else if (plan.max_reach <= 1) {
    const size_t sm_fill = cellscan_smem(true);
    prefer_shared(k_cellscan<true>, sm_fill);
    k_cellscan<true><<<dim3((unsigned)plan.ncell_cap, (unsigned)nsplit), kScanWarps * 32,
                       sm_fill, stream>>>(a);
  } else {
    const size_t fill_smem = (size_t)kFillWarps * 2 * kFillMaxCand * sizeof(unsigned long long);
    k_fill<<<(int)((a.n + kFillWarps - 1) / kFillWarps), kFillWarps * 32, fill_smem, stream>>>(
        a);
  }
}

// The one-launch build with stage capacity CAP; MLG_ERR_UNSUPPORTED if the
// driver refuses the cooperative launch (the caller then runs the chain).
template <int CAP>
int launch_fused_build(const BuildArgs& a, const BuildPlan& plan, int nsplit, FusedSync* sync,
                       cudaStream_t stream) {
  const int64_t n = a.n;
  const size_t smem = fused_build_smem<CAP>(n);
  auto kern = k_build_fused<CAP>;
  prefer_shared(kern, smem);
  const int64_t cap = (int64_t)resident_blocks(kern, kCellWarps * 32, smem) * sm_count();
  const int64_t nitems = (int64_t)plan.ncell_cap * nsplit;
  const int grid = (int)(nitems < cap ? nitems : cap);
  if (cudaMemsetAsync(sync, 0, sizeof(FusedSync), stream) != cudaSuccess) return MLG_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kCellWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, a, plan, plan.ncell_cap, nsplit, sync) == cudaSuccess)
    return launch_status();
  (void)cudaGetLastError();
  return MLG_ERR_UNSUPPORTED;
}

// Options of a build beyond mlg_build_csr's arguments.
struct BuildOptions {
  const uint32_t* gate = nullptr;  // device word: 0 = every kernel returns at once
  bool wait_test = false;          // one-launch build only, with the two knobs below
  long long polls = 0;             // polls of each bounded wait before it gives up
  int hold_release = 0;            // CTA 0 never releases the binned atoms
};

int build_impl(const mlg_system* sys, double rcut, double r_on, int32_t nnei_max,
               const mlg_csr* csr, void* ws, size_t ws_bytes, cudaStream_t stream,
               const BuildOptions& opt = BuildOptions()) {
  if (sys == nullptr || sys->coords == nullptr) return MLG_ERR_INVALID_ARG;
  if (sys->types != nullptr && sys->n_types < 1) return MLG_ERR_INVALID_ARG;
  int rc = check_build_args(rcut, r_on, nnei_max, csr);
  if (rc != MLG_OK) return rc;
  BuildPlan plan;
  rc = make_plan(sys->n_atoms, rcut, sys->box, sys->pbc, &plan);
  if (rc != MLG_OK) return rc;
  const int64_t n = sys->n_atoms;
  BuildLayout L = build_layout(n, plan.ncell_cap);
  if (ws == nullptr || ws_bytes < L.total || ((uintptr_t)ws % kAlign) != 0)
    return MLG_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  BuildArgs a = make_build_args(sys, rcut, r_on, nnei_max, csr, w, L);
  const int nsplit = build_nsplit(plan);
  a.gate = opt.gate;
  if (opt.wait_test) {
    if (!use_fused_build(plan, n)) return MLG_ERR_UNSUPPORTED;
    a.spin_polls = opt.polls;
    a.hold_release = opt.hold_release;
  }
  // the key stash of the count-to-fill chain, when the workspace holds it
  if (!use_fused_build(plan, n) && plan.max_reach <= 1 && ws_bytes >= L.total_stash) {
    a.stash = reinterpret_cast<unsigned long long*>(w + L.stash);
    a.stash_n = reinterpret_cast<int*>(w + L.stash_n);
    a.stash_q = n <= (int64_t(1) << 21) ? 1 : 0;
  }
  if (use_fused_build(plan, n)) {
    // the whole build in one cooperative launch (small systems); systems of
    // at most 75 atoms take the larger stage, which holds any 27-cell stencil
    // (27 n candidates) so that no centre takes the global-memory traversal
    FusedSync* sync = reinterpret_cast<FusedSync*>(w + L.sync);
    const int rc2 = 27 * n <= kCellCandSmall
                        ? launch_fused_build<kCellCandSmall>(a, plan, nsplit, sync, stream)
                        : launch_fused_build<kCellCand>(a, plan, nsplit, sync, stream);
    if (rc2 != MLG_ERR_UNSUPPORTED || opt.wait_test) return rc2;
    // refused (not co-resident): the kernel chain below
  }
  launch_count_phase(a, plan, nsplit, stream);
  launch_scan<long long>(a.kept, n, reinterpret_cast<long long*>(a.row_ptr), a.partial,
                         ScanTail{a.n_edges, a.status, a.capacity, a.gate}, stream);
  launch_fill_phase(a, plan, nsplit, stream);
  return launch_status();
}

// ---------------------------------------------------------------- batches
//
// Workspace of a batch: the kept and raw counts of all atoms (one array, so
// that one scan gives the global row starts) and its scan partials, then the
// build workspace of each system with atoms.
struct BatchTotals {
  int64_t n_total;
  size_t global_bytes;
  size_t total;
  size_t kept, raw, partial;
};

int batch_totals(const mlg_system* systems, int32_t n_systems, double rcut, BatchTotals* t) {
  if (n_systems < 0 || (n_systems > 0 && systems == nullptr)) return MLG_ERR_INVALID_ARG;
  int64_t n_total = 0;
  size_t per_sys = 0;
  for (int32_t k = 0; k < n_systems; ++k) {
    const mlg_system& s = systems[k];
    if (s.n_atoms < 0) return MLG_ERR_INVALID_ARG;
    if (s.n_atoms == 0) continue;
    if (s.coords == nullptr || (s.types != nullptr && s.n_types < 1)) return MLG_ERR_INVALID_ARG;
    BuildPlan plan;
    int rc = make_plan(s.n_atoms, rcut, s.box, s.pbc, &plan);
    if (rc != MLG_OK) return rc;
    per_sys += align_up(build_layout(s.n_atoms, plan.ncell_cap).total);
    n_total += s.n_atoms;
  }
  if (n_total > (int64_t)INT32_MAX / 2) return MLG_ERR_UNSUPPORTED;
  t->n_total = n_total;
  size_t off = 0;
  t->kept = off;
  off = align_up(off + (size_t)n_total * sizeof(int));
  t->raw = off;
  off = align_up(off + (size_t)n_total * sizeof(int));
  t->partial = off;
  off = align_up(off + (size_t)(scan_tiles(n_total > 0 ? n_total : 1) + 2) * sizeof(long long));
  t->global_bytes = off;
  t->total = off + per_sys;
  return MLG_OK;
}

int build_batch_impl(const mlg_system* systems, int32_t n_systems, double rcut, double r_on,
                     int32_t nnei_max, const mlg_csr* csr, void* ws, size_t ws_bytes,
                     cudaStream_t stream) {
  int rc = check_build_args(rcut, r_on, nnei_max, csr);
  if (rc != MLG_OK) return rc;
  BatchTotals T;
  rc = batch_totals(systems, n_systems, rcut, &T);
  if (rc != MLG_OK) return rc;
  if (ws == nullptr || ws_bytes < T.total || ((uintptr_t)ws % kAlign) != 0)
    return MLG_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  int* kept = reinterpret_cast<int*>(w + T.kept);
  int* raw = reinterpret_cast<int*>(w + T.raw);
  long long* partial = reinterpret_cast<long long*>(w + T.partial);
  if (cudaMemsetAsync(csr->status, 0, sizeof(uint32_t), stream) != cudaSuccess ||
      cudaMemsetAsync(csr->n_truncated, 0, sizeof(int64_t), stream) != cudaSuccess)
    return MLG_ERR_CUDA;
  // count every system into its slice of the kept counts
  for (int pass = 0; pass < 2; ++pass) {
    if (pass == 1)
      launch_scan<long long>(kept, T.n_total, reinterpret_cast<long long*>(csr->row_ptr),
                             partial, ScanTail{csr->n_edges, csr->status, csr->capacity},
                             stream);
    size_t sys_off = T.global_bytes;
    int64_t atom_off = 0;
    for (int32_t k = 0; k < n_systems; ++k) {
      const mlg_system& s = systems[k];
      if (s.n_atoms == 0) continue;
      BuildPlan plan;
      make_plan(s.n_atoms, rcut, s.box, s.pbc, &plan);
      const BuildLayout L = build_layout(s.n_atoms, plan.ncell_cap);
      BuildArgs a = make_build_args(&s, rcut, r_on, nnei_max, csr, w + sys_off, L);
      a.kept = kept + atom_off;
      a.raw = raw + atom_off;
      a.row_ptr = csr->row_ptr + atom_off;
      a.src_offset = (int32_t)atom_off;
      a.zero_globals = 0;
      if (pass == 0)
        launch_count_phase(a, plan, build_nsplit(plan), stream);
      else
        launch_fill_phase(a, plan, build_nsplit(plan), stream);
      sys_off += align_up(L.total);
      atom_off += s.n_atoms;
    }
  }
  return launch_status();
}

int sm_count() {
  static int cached[64] = {0};
  const int dev = current_device();
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cached[dev] = sms;
  return sms;
}

// One layer of the generic kernel over the centres with more than min_n edges.
int launch_generic(const mlg_csr* csr, int64_t n_centres, int32_t nnei_max, int32_t C, int32_t H,
                   mlg_dtype dtype, const void* G_in, void* G_out, const void* Wq,
                   const void* Wk, const void* Wv, int min_n, cudaStream_t stream,
                   int smooth = 0) {
  AttnArgs a;
  a.row_ptr = csr->row_ptr;
  a.sw = csr->sw;
  a.n_centres = n_centres;
  a.capacity = csr->capacity;
  a.nnei_max = nnei_max;
  a.C = C;
  a.H = H;
  a.D = C / H;
  a.G = G_in;
  a.out = G_out;
  a.Wq = Wq;
  a.Wk = Wk;
  a.Wv = Wv;
  a.status = csr->status;
  a.min_n = min_n;
  a.smooth = smooth;
  int64_t want = (int64_t)sm_count() * 4;
  int grid = (int)(n_centres < want ? n_centres : want);
  if (dtype == MLG_F64) {
    size_t smem = attn_generic_smem<double>(nnei_max, a.D);
    if (smem > 227 * 1024) return MLG_ERR_UNSUPPORTED;
    prefer_shared(k_attn_generic<double>, smem);
    k_attn_generic<double><<<grid, kAttnWarps * 32, smem, stream>>>(a);
  } else {
    size_t smem = attn_generic_smem<float>(nnei_max, a.D);
    if (smem > 227 * 1024) return MLG_ERR_UNSUPPORTED;
    prefer_shared(k_attn_generic<float>, smem);
    k_attn_generic<float><<<grid, kAttnWarps * 32, smem, stream>>>(a);
  }
  return launch_status();
}

// FP64 tensor-core kernel: one CTA of NT threads per SM (shared memory), tiles
// of R rows, centres of at most 8 NBC edges.
template <int R, int NBC, int NT>
int launch_dmma(TileArgs& ta, cudaStream_t stream) {
  using Cfg = DmmaCfg<R, NBC, NT>;
  auto kern = k_attn_dmma<R, NBC, NT>;
  prefer_shared(kern, Cfg::SMEM);
  if (cudaGetLastError() != cudaSuccess) return MLG_ERR_CUDA;
  int occ = resident_blocks(kern, NT, Cfg::SMEM);
  int64_t want = (int64_t)sm_count() * occ;
  int grid = (int)(ta.n_centres < want ? ta.n_centres : want);
  if (grid < 1) grid = 1;
  kern<<<grid, NT, Cfg::SMEM, stream>>>(ta);
  return launch_status();
}

// A 2-D tensor map over G [rows][C] fp32 with a {4 x 128} box (16-byte inner
// extent), for the tcgen05 kernel's slab loads.  Encoded on the host per call
// (no device work, no allocation).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode_slab_map(CUtensorMap* map, const void* G, int64_t rows, int C, int box_rows = 128) {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  const cuuint64_t dims[2] = {(cuuint64_t)C, (cuuint64_t)(rows > 0 ? rows : 1)};
  const cuuint64_t strides[1] = {(cuuint64_t)C * 4};
  const cuuint32_t box[2] = {4, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(G), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32, 32 or 64 channels: projection on tcgen05 (3xTF32), tiles of 128 rows.
// TMEM columns per CTA: 128 (c = 32) or 256 (c = 64); the grid keeps the
// resident CTAs within the 512 columns of an SM.
template <int C, int D, int NT>
int launch_tc(TileArgs& ta, cudaStream_t stream) {
  using Cfg = TcCfg<C, D, NT>;
  auto kern = k_attn_tc<C, D, NT>;
  prefer_shared(kern, Cfg::SMEM);
  if (cudaGetLastError() != cudaSuccess) return MLG_ERR_CUDA;
  CUtensorMap map;
  if (!encode_slab_map(&map, ta.G, ta.capacity, C)) return MLG_ERR_CUDA;
  int occ = resident_blocks(kern, NT, Cfg::SMEM);
  const int tmem_cap = 512 / Cfg::NCOL;
  if (occ > tmem_cap) occ = tmem_cap;
  int64_t want = (int64_t)sm_count() * occ;
  int grid = (int)(ta.n_centres < want ? ta.n_centres : want);
  if (grid < 1) grid = 1;
  kern<<<grid, NT, Cfg::SMEM, stream>>>(ta, map);
  return launch_status();
}

// fp32, 32 channels, 4 heads, one layer, centres of up to 64 edges: one CTA
// per SM holding all of its TMEM.  Which kernel takes these rows (a build-time
// choice for A/B runs): 0 = the tile kernel of every fp32 row (logits and P V
// on the FP32 pipe), 2 = every product on tcgen05, 6 = the logits on tcgen05
// with one 64-column TMEM buffer per head and P V on the FP32 pipe, 7 = as 6
// with P V on warp-level tensor-core MMAs and the slabs planned and loaded two
// tiles ahead.
#ifndef MLG_TC_ATTN
#define MLG_TC_ATTN 7
#endif
constexpr bool kTcAttn = MLG_TC_ATTN != 0;
int launch_tc2(TileArgs& ta, cudaStream_t stream) {
#if MLG_TC_ATTN == 7
  auto kern = k_attn_tc7;
  const size_t smem = tc7::SMEM;
  const int nt = tc7::NT;
#elif MLG_TC_ATTN == 6
  auto kern = k_attn_tc6;
  const size_t smem = tc6::SMEM;
  const int nt = tc6::NT;
#else
  auto kern = k_attn_tc2;
  const size_t smem = tc2::SMEM;
  const int nt = tc2::NT;
#endif
  prefer_shared(kern, smem);
  if (cudaGetLastError() != cudaSuccess) return MLG_ERR_CUDA;
  CUtensorMap map;
  if (!encode_slab_map(&map, ta.G, ta.capacity, tc2::C, 32)) return MLG_ERR_CUDA;
  const int64_t want = sm_count();
  int grid = (int)(ta.n_centres < want ? ta.n_centres : want);
  if (grid < 1) grid = 1;
  kern<<<grid, nt, smem, stream>>>(ta, map);
  return launch_status();
}

// fp64, 32 channels, head size 8: FP64 tensor-core kernel; the most edges of
// a centre it takes (40 or 64), by nnei_max
int dmma_rows(int nnei_max) { return nnei_max <= 40 ? 40 : 64; }

// Returns the most edges of a centre that the fused kernel for this shape
// takes (0: no fused kernel); larger centres go to the generic kernel.
int tile_rows(mlg_dtype dtype, int C, int D, int nnei_max) {
  if (dtype == MLG_F64 && C == 32 && D == 8) return dmma_rows(nnei_max);
  if (dtype == MLG_F32 && C == 32 && D == 8) return 128;
  if (dtype == MLG_F32 && C == 64 && D == 16) return 128;
  return 0;
}

int launch_tile_shape(mlg_dtype dtype, int C, int D, int nnei_max, TileArgs& ta,
                      cudaStream_t s) {
  if (dtype == MLG_F64 && C == 32 && D == 8)
    return dmma_rows(nnei_max) == 40 ? launch_dmma<160, 5, 640>(ta, s)
                                     : launch_dmma<128, 8, 512>(ta, s);
  if (dtype == MLG_F32 && C == 32 && D == 8) return launch_tc<32, 8, 512>(ta, s);
  if (dtype == MLG_F32 && C == 64 && D == 16) return launch_tc<64, 16, 512>(ta, s);
  return MLG_ERR_UNSUPPORTED;
}

// Head-group kernel instantiations for wide features: (dtype, channels, head size) -> R.
template <typename T, int C, int D, int HG, int R, int NT, int TM, int TN, int KC>
int launch_hg(HgArgs& ha, cudaStream_t stream) {
  using Cfg = HgCfg<T, C, D, HG, R, NT, TM, TN, KC>;
  auto kern = k_attn_hg<T, C, D, HG, R, NT, TM, TN, KC>;
  prefer_shared(kern, Cfg::SMEM);
  if (cudaGetLastError() != cudaSuccess) return MLG_ERR_CUDA;
  const int occ = resident_blocks(kern, NT, Cfg::SMEM);
  int64_t gx = ((int64_t)sm_count() * occ + Cfg::NG - 1) / Cfg::NG;
  if (gx > ha.n_centres) gx = ha.n_centres;
  if (gx < 1) gx = 1;
  kern<<<dim3((unsigned)gx, Cfg::NG), NT, Cfg::SMEM, stream>>>(ha);
  return launch_status();
}

int hg_rows(mlg_dtype dtype, int C, int D) {
  if (dtype == MLG_F64 && C == 128 && D == 32) return 128;
  if (dtype == MLG_F32 && C == 128 && D == 16) return hgtc::R;
  return 0;
}

// fp32, 128 channels, heads of 16: the projection on tcgen05, grid (centre
// ranges x 4 head groups), one CTA per SM.
int launch_hgtc(const HgArgs& ha, cudaStream_t stream) {
  auto kern = k_attn_hgtc;
  prefer_shared(kern, hgtc::SMEM);
  if (cudaGetLastError() != cudaSuccess) return MLG_ERR_CUDA;
  CUtensorMap map;
  if (!encode_slab_map(&map, ha.G, ha.capacity, hgtc::C, 128)) return MLG_ERR_CUDA;
  HgtcArgs a;
  a.row_ptr = ha.row_ptr;
  a.sw = ha.sw;
  a.n_centres = ha.n_centres;
  a.capacity = ha.capacity;
  a.nnei_max = ha.nnei_max;
  a.smooth = ha.smooth;
  a.out = ha.out;
  a.Wq = ha.Wq;
  a.Wk = ha.Wk;
  a.Wv = ha.Wv;
  a.status = ha.status;
  int64_t gx = ((int64_t)sm_count() + hgtc::NG - 1) / hgtc::NG;
  if (gx > ha.n_centres) gx = ha.n_centres;
  if (gx < 1) gx = 1;
  kern<<<dim3((unsigned)gx, hgtc::NG), hgtc::NT, hgtc::SMEM, stream>>>(a, map);
  return launch_status();
}

int launch_hg_shape(mlg_dtype dtype, int C, int D, HgArgs& ha, cudaStream_t s) {
  if (dtype == MLG_F64 && C == 128 && D == 32)
    return launch_hg<double, 128, 32, 1, 128, 256, 8, 6, 16>(ha, s);
  if (dtype == MLG_F32 && C == 128 && D == 16) return launch_hgtc(ha, s);
  return MLG_ERR_UNSUPPORTED;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int check_attention_args(const mlg_csr* csr, int64_t n_centres, int32_t nnei_max,
                         int32_t channels, int32_t heads, mlg_dtype dtype, const void* G_in,
                         void* G_out) {
  if (csr == nullptr || csr->row_ptr == nullptr || csr->sw == nullptr || csr->status == nullptr)
    return MLG_ERR_INVALID_ARG;
  if (n_centres < 0 || nnei_max < 1 || channels < 1 || heads < 1 || channels % heads != 0)
    return MLG_ERR_INVALID_ARG;
  if (!G_in || !G_out) return MLG_ERR_INVALID_ARG;
  if (G_in == G_out) return MLG_ERR_INVALID_ARG;
  if (dtype != MLG_F32 && dtype != MLG_F64) return MLG_ERR_INVALID_ARG;
  const int D = channels / heads;
  if (nnei_max > kMaxNnei || channels > 256 || D > 64) return MLG_ERR_UNSUPPORTED;
  return MLG_OK;
}

// n_layers attention layers G^{l+1} = attention(G^l), G^0 = G_in, result in
// G_out.  `pong` is a [capacity][channels] buffer, needed only for
// n_layers >= 2 on the generic path.  With `smooth`, every layer uses the
// slot-occupancy softmax (phantom slots up to nnei_max); the FP64 tensor-core
// kernel has no such variant, so that shape runs on the generic kernel.
int attention_stack_impl(const mlg_csr* csr, int64_t n_centres, int32_t nnei_max,
                         int32_t channels, int32_t heads, mlg_dtype dtype, int32_t n_layers,
                         const void* const* W, const void* G_in, void* G_out, void* pong,
                         cudaStream_t stream, int smooth = 0) {
  int rc = check_attention_args(csr, n_centres, nnei_max, channels, heads, dtype, G_in, G_out);
  if (rc != MLG_OK) return rc;
  if (n_layers < 1 || W == nullptr) return MLG_ERR_INVALID_ARG;
  for (int k = 0; k < 3 * n_layers; ++k)
    if (W[k] == nullptr) return MLG_ERR_INVALID_ARG;
  if (n_layers >= 2 && pong == nullptr) return MLG_ERR_WORKSPACE;
  if (n_centres == 0) return MLG_OK;
  const int D = channels / heads;
  int R = tile_rows(dtype, channels, D, nnei_max);
  if (smooth && dtype == MLG_F64) R = 0;  // no slot-occupancy FP64 tensor-core kernel
  bool tile_ok = R > 0 && n_layers <= kMaxFusedLayers && aligned16(G_in) && aligned16(G_out);
  for (int k = 0; tile_ok && k < 3 * n_layers; ++k) tile_ok = aligned16(W[k]);
  int min_n = 0;  // generic path: centres with more than min_n edges
  if (tile_ok) {
    TileArgs ta;
    std::memset(&ta, 0, sizeof(ta));
    ta.row_ptr = csr->row_ptr;
    ta.sw = csr->sw;
    ta.n_centres = n_centres;
    ta.capacity = csr->capacity;
    ta.n_layers = n_layers;
    ta.nnei_max = nnei_max;
    ta.smooth = smooth;
    ta.G = G_in;
    ta.out = G_out;
    for (int k = 0; k < 3 * n_layers; ++k) ta.W[k] = W[k];
    ta.status = csr->status;
    if (kTcAttn && dtype == MLG_F32 && channels == 32 && D == 8 && n_layers == 1) {
      // centres of up to 64 edges with every product on tcgen05; longer ones
      // (up to the tile) on the kernel whose logits and P V run on the FP32 pipe
      rc = launch_tc2(ta, stream);
      if (rc != MLG_OK) return rc;
      if (nnei_max > tc2::MAXN) {
        ta.min_n = tc2::MAXN;
        rc = launch_tile_shape(dtype, channels, D, nnei_max, ta, stream);
        if (rc != MLG_OK) return rc;
      }
    } else {
      rc = launch_tile_shape(dtype, channels, D, nnei_max, ta, stream);
      if (rc != MLG_OK) return rc;
    }
    if (nnei_max <= R) return MLG_OK;  // no centre can exceed the tile
    min_n = R;
  }
  // head-group kernel (one launch per layer) when there is one for the shape
  int Rg = tile_ok ? 0 : hg_rows(dtype, channels, D);
  bool hg_ok = Rg > 0 && aligned16(G_in) && aligned16(G_out) && (n_layers < 2 || aligned16(pong));
  for (int k = 0; hg_ok && k < 3 * n_layers; ++k) hg_ok = aligned16(W[k]);
  if (hg_ok) min_n = nnei_max <= Rg ? -1 : Rg;  // -1: no generic launch needed
  // per layer: head-group kernel and/or the generic kernel for the centres left
  const void* in = G_in;
  for (int l = 0; l < n_layers; ++l) {
    void* dst = ((n_layers - 1 - l) % 2 == 0) ? G_out : pong;
    if (hg_ok) {
      HgArgs ha;
      ha.row_ptr = csr->row_ptr;
      ha.sw = csr->sw;
      ha.n_centres = n_centres;
      ha.capacity = csr->capacity;
      ha.nnei_max = nnei_max;
      ha.smooth = smooth;
      ha.G = in;
      ha.out = dst;
      ha.Wq = W[3 * l];
      ha.Wk = W[3 * l + 1];
      ha.Wv = W[3 * l + 2];
      ha.status = csr->status;
      rc = launch_hg_shape(dtype, channels, D, ha, stream);
      if (rc != MLG_OK) return rc;
    }
    if (min_n >= 0) {
      rc = launch_generic(csr, n_centres, nnei_max, channels, heads, dtype, in, dst, W[3 * l],
                          W[3 * l + 1], W[3 * l + 2], min_n, stream, smooth);
      if (rc != MLG_OK) return rc;
    }
    in = dst;
  }
  return MLG_OK;
}

// Workspace of mlg_verlet_step: the list build's workspace (at rcut + skin),
// the check's scratch words, the refine's per-destination counts and scan
// partials.
struct VerletLayout {
  size_t build_bytes, scratch, kept, raw, partial, total;
};

int verlet_layout(int64_t n, double rcut, double skin, const double* box, const uint8_t* pbc,
                  VerletLayout* V) {
  if (!(skin >= 0.0) || !std::isfinite(skin)) return MLG_ERR_INVALID_ARG;
  BuildPlan plan;
  int rc = make_plan(n, rcut + skin, box, pbc, &plan);
  if (rc != MLG_OK) return rc;
  size_t off = align_up(build_layout(n, plan.ncell_cap).total);
  V->build_bytes = off;
  V->scratch = off;
  off = align_up(off + 16);
  V->kept = off;
  off = align_up(off + (size_t)n * sizeof(int));
  V->raw = off;
  off = align_up(off + (size_t)n * sizeof(int));
  V->partial = off;
  off = align_up(off + (size_t)(scan_tiles(n) + 2) * sizeof(long long));
  V->total = off;
  return MLG_OK;
}

int verlet_step_impl(const mlg_system* sys, double rcut, double r_on, double skin,
                     int32_t nnei_max, const mlg_verlet_list* list, const mlg_csr* out, void* ws,
                     size_t ws_bytes, cudaStream_t stream) {
  if (sys == nullptr || sys->coords == nullptr || list == nullptr) return MLG_ERR_INVALID_ARG;
  if (list->coords_ref == nullptr || list->state == nullptr || list->n_builds == nullptr)
    return MLG_ERR_INVALID_ARG;
  if (sys->types != nullptr && sys->n_types < 1) return MLG_ERR_INVALID_ARG;
  int rc = check_build_args(rcut, r_on, nnei_max, out);
  if (rc != MLG_OK) return rc;
  rc = check_csr(&list->cand);
  if (rc != MLG_OK) return rc;
  const int64_t n = sys->n_atoms;
  VerletLayout V;
  rc = verlet_layout(n, rcut, skin, sys->box, sys->pbc, &V);
  if (rc != MLG_OK) return rc;
  if (ws == nullptr || ws_bytes < V.total || ((uintptr_t)ws % kAlign) != 0)
    return MLG_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  uint32_t* gate = reinterpret_cast<uint32_t*>(w + V.scratch);
  if (cudaMemsetAsync(gate, 0, 16, stream) != cudaSuccess) return MLG_ERR_CUDA;
  // 1. the displacement check decides on the device whether the list is rebuilt
  VerletCheckArgs ca;
  ca.n = n;
  ca.coords = sys->coords;
  ca.coords_ref = list->coords_ref;
  ca.state = list->state;
  ca.skin = skin;
  ca.gate = gate;
  ca.done = reinterpret_cast<unsigned int*>(gate + 1);
  ca.dmax = reinterpret_cast<unsigned long long*>(w + V.scratch + 8);
  ca.out_status = out->status;
  ca.out_trunc = out->n_truncated;
  const int64_t cblocks = (n + 255) / 256;
  const int64_t cmax = (int64_t)sm_count() * 4;
  k_verlet_check<<<(unsigned)(cblocks < cmax ? cblocks : cmax), 256, 0, stream>>>(ca);
  // 2. the list's build, gated on that decision, and its coordinates
  BuildOptions opt;
  opt.gate = gate;
  rc = build_impl(sys, rcut + skin, r_on, kVerletListCap, &list->cand, w, V.build_bytes, stream,
                  opt);
  if (rc != MLG_OK) return rc;
  const int64_t t3 = (3 * n + 255) / 256;
  k_verlet_commit<<<(unsigned)(t3 < cmax ? t3 : cmax), 256, 0, stream>>>(
      gate, n, sys->coords, list->coords_ref, list->state, list->n_builds);
  // 3. the refine: count, scan, fill
  RefineArgs ra;
  std::memset(&ra, 0, sizeof(ra));
  ra.n = n;
  ra.coords = sys->coords;
  std::memcpy(ra.box, sys->box, sizeof(ra.box));
  ra.rcut = rcut;
  ra.r_on = r_on;
  ra.rc2 = rcut * rcut;
  ra.nnei_max = nnei_max;
  taylor_coeffs(ra.taylor);
  ra.cp = list->cand.row_ptr;
  ra.cs = list->cand.src;
  ra.ch = list->cand.shift;
  ra.cand_status = list->cand.status;
  ra.cand_trunc = list->cand.n_truncated;
  ra.kept = reinterpret_cast<int*>(w + V.kept);
  ra.raw = reinterpret_cast<int*>(w + V.raw);
  ra.capacity = out->capacity;
  ra.row_ptr = out->row_ptr;
  ra.src = out->src;
  ra.shift = out->shift;
  ra.vec = out->vec;
  ra.dist = out->dist;
  ra.sw = out->sw;
  ra.n_truncated = out->n_truncated;
  ra.status = out->status;
  const unsigned rblocks = (unsigned)((n + kRefineWarps - 1) / kRefineWarps);
  k_refine_count<<<rblocks, kRefineWarps * 32, 0, stream>>>(ra);
  launch_scan<long long>(ra.kept, n, reinterpret_cast<long long*>(out->row_ptr),
                         reinterpret_cast<long long*>(w + V.partial),
                         ScanTail{out->n_edges, out->status, out->capacity, nullptr}, stream);
  k_refine_fill<<<rblocks, kRefineWarps * 32, 0, stream>>>(ra);
  return launch_status();
}

int forward_launches(int64_t n_atoms, int32_t nnei_max, int32_t channels, int32_t heads,
                     int32_t n_layers, mlg_dtype dtype) {
  const int D = heads > 0 ? channels / heads : 0;
  int R = tile_rows(dtype, channels, D, nnei_max);
  if (R > 0 && n_layers <= kMaxFusedLayers) {
    const bool tc2_path =
        kTcAttn && dtype == MLG_F32 && channels == 32 && D == 8 && n_layers == 1;
    return 1 + (tc2_path && nnei_max > tc2::MAXN ? 1 : 0) + (nnei_max > R ? n_layers : 0);
  }
  int Rg = hg_rows(dtype, channels, D);
  if (Rg > 0) return n_layers * (1 + (nnei_max > Rg ? 1 : 0));
  (void)n_atoms;
  return n_layers;
}

}  // namespace

extern "C" {

size_t mlg_build_csr_workspace_bytes(int64_t n_atoms, double rcut, const double box[9],
                                     const uint8_t pbc[3]) {
  BuildPlan plan;
  if (make_plan(n_atoms, rcut, box, pbc, &plan) != MLG_OK) return 0;
  const BuildLayout L = build_layout(n_atoms, plan.ncell_cap);
  // the key stash only where the kernel chain with per-cell scans runs
  return !use_fused_build(plan, n_atoms) && plan.max_reach <= 1 ? L.total_stash : L.total;
}

int mlg_build_csr(const mlg_system* sys, double rcut, double r_on, int32_t nnei_max,
                  const mlg_csr* csr, void* ws, size_t ws_bytes, mlg_stream_t stream) {
  return build_impl(sys, rcut, r_on, nnei_max, csr, ws, ws_bytes, (cudaStream_t)stream);
}

size_t mlg_build_csr_batch_workspace_bytes(const mlg_system* systems, int32_t n_systems,
                                           double rcut) {
  if (!(rcut > 0.0) || !std::isfinite(rcut)) return 0;
  BatchTotals T;
  if (batch_totals(systems, n_systems, rcut, &T) != MLG_OK) return 0;
  return T.total;
}

int mlg_build_csr_batch(const mlg_system* systems, int32_t n_systems, double rcut, double r_on,
                        int32_t nnei_max, const mlg_csr* csr, void* ws, size_t ws_bytes,
                        mlg_stream_t stream) {
  return build_batch_impl(systems, n_systems, rcut, r_on, nnei_max, csr, ws, ws_bytes,
                          (cudaStream_t)stream);
}

size_t mlg_attention_workspace_bytes(int64_t n_centres, int32_t nnei_max, int32_t channels,
                                     int32_t heads, mlg_dtype dtype) {
  (void)n_centres;
  (void)nnei_max;
  (void)channels;
  (void)heads;
  (void)dtype;
  return 0;
}

int mlg_block_attention(const mlg_csr* csr, int64_t n_centres, int32_t nnei_max,
                        int32_t channels, int32_t heads, mlg_dtype dtype, const void* G_in,
                        void* G_out, const void* Wq, const void* Wk, const void* Wv, void* ws,
                        size_t ws_bytes, mlg_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  const void* W[3] = {Wq, Wk, Wv};
  if (!Wq || !Wk || !Wv) return MLG_ERR_INVALID_ARG;
  return attention_stack_impl(csr, n_centres, nnei_max, channels, heads, dtype, 1, W, G_in, G_out,
                              nullptr, (cudaStream_t)stream);
}

int mlg_local_attention(const mlg_csr* csr, int64_t n_centres, int32_t nnei_max,
                        int32_t channels, int32_t heads, mlg_dtype dtype, const void* H_in,
                        const void* G_in, void* out, const void* Wq, const void* Wk,
                        const void* Wv, mlg_stream_t stream) {
  int rc = check_attention_args(csr, n_centres, nnei_max, channels, heads, dtype, G_in, out);
  if (rc != MLG_OK) return rc;
  if (H_in == nullptr || H_in == out || !Wq || !Wk || !Wv) return MLG_ERR_INVALID_ARG;
  if (n_centres == 0) return MLG_OK;
  if (channels > kLocalMaxC) return MLG_ERR_UNSUPPORTED;
  LocalArgs la;
  la.row_ptr = csr->row_ptr;
  la.sw = csr->sw;
  la.n_centres = n_centres;
  la.capacity = csr->capacity;
  la.channels = channels;
  la.heads = heads;
  la.nnei_max = nnei_max;
  la.H = H_in;
  la.G = G_in;
  la.out = out;
  la.Wq = Wq;
  la.Wk = Wk;
  la.Wv = Wv;
  la.status = csr->status;
  cudaStream_t st = (cudaStream_t)stream;
  auto go = [&](auto kern, size_t smem) {
    if (smem > 227 * 1024) return (int)MLG_ERR_UNSUPPORTED;
    prefer_shared(kern, smem);
    if (cudaGetLastError() != cudaSuccess) return (int)MLG_ERR_CUDA;
    const int64_t want = (int64_t)resident_blocks(kern, kLocalThreads, smem) * sm_count();
    const int grid = (int)(n_centres < want ? n_centres : want);
    kern<<<grid, kLocalThreads, smem, st>>>(la);
    return launch_status();
  };
  // 32 channels: one warp per centre
  auto go_w32 = [&](auto kern, size_t smem) {
    if (smem > 227 * 1024) return (int)MLG_ERR_UNSUPPORTED;
    prefer_shared(kern, smem);
    if (cudaGetLastError() != cudaSuccess) return (int)MLG_ERR_CUDA;
    const int nt = kLocalW32Warps * 32;
    const int64_t want = (int64_t)resident_blocks(kern, nt, smem) * sm_count();
    const int64_t need = (n_centres + kLocalW32Warps - 1) / kLocalW32Warps;
    const int grid = (int)(need < want ? need : want);
    kern<<<grid < 1 ? 1 : grid, nt, smem, st>>>(la);
    return launch_status();
  };
  if (channels == 32 && (heads == 1 || heads == 2 || heads == 4 || heads == 8)) {
    const bool f64 = dtype == MLG_F64;
    switch (heads) {
      case 1: return f64 ? go_w32(k_local_attn_w32<double, 1>, local_w32_smem<double, 1>(nnei_max))
                         : go_w32(k_local_attn_w32<float, 1>, local_w32_smem<float, 1>(nnei_max));
      case 2: return f64 ? go_w32(k_local_attn_w32<double, 2>, local_w32_smem<double, 2>(nnei_max))
                         : go_w32(k_local_attn_w32<float, 2>, local_w32_smem<float, 2>(nnei_max));
      case 4: return f64 ? go_w32(k_local_attn_w32<double, 4>, local_w32_smem<double, 4>(nnei_max))
                         : go_w32(k_local_attn_w32<float, 4>, local_w32_smem<float, 4>(nnei_max));
      default: return f64 ? go_w32(k_local_attn_w32<double, 8>, local_w32_smem<double, 8>(nnei_max))
                          : go_w32(k_local_attn_w32<float, 8>, local_w32_smem<float, 8>(nnei_max));
    }
  }
  if (dtype == MLG_F64)
    return go(k_local_attn<double>, local_smem<double>(channels, heads, nnei_max));
  return go(k_local_attn<float>, local_smem<float>(channels, heads, nnei_max));
}

int mlg_block_attention_smooth(const mlg_csr* csr, int64_t n_centres, int32_t nnei_max,
                               int32_t channels, int32_t heads, mlg_dtype dtype,
                               const void* G_in, void* G_out, const void* Wq, const void* Wk,
                               const void* Wv, mlg_stream_t stream) {
  int rc = check_attention_args(csr, n_centres, nnei_max, channels, heads, dtype, G_in, G_out);
  if (rc != MLG_OK) return rc;
  if (!Wq || !Wk || !Wv) return MLG_ERR_INVALID_ARG;
  const void* W[3] = {Wq, Wk, Wv};
  return attention_stack_impl(csr, n_centres, nnei_max, channels, heads, dtype, 1, W, G_in, G_out,
                              nullptr, (cudaStream_t)stream, 1);
}

size_t mlg_attention_stack_workspace_bytes(int64_t capacity, int32_t channels, int32_t n_layers,
                                           mlg_dtype dtype) {
  if (capacity < 0 || channels < 1 || n_layers < 1) return 0;
  size_t el = dtype == MLG_F64 ? 8 : 4;
  return n_layers >= 2 ? align_up((size_t)(capacity > 0 ? capacity : 1) * channels * el) : 0;
}

int mlg_attention_stack_smooth(const mlg_csr* csr, int64_t n_centres, int32_t nnei_max,
                               int32_t channels, int32_t heads, int32_t n_layers,
                               mlg_dtype dtype, const void* const* W, const void* G_in,
                               void* G_out, void* ws, size_t ws_bytes, mlg_stream_t stream) {
  if (csr == nullptr) return MLG_ERR_INVALID_ARG;
  size_t need = mlg_attention_stack_workspace_bytes(csr->capacity, channels, n_layers, dtype);
  if (need > 0 && (ws == nullptr || ws_bytes < need)) return MLG_ERR_WORKSPACE;
  return attention_stack_impl(csr, n_centres, nnei_max, channels, heads, dtype, n_layers, W, G_in,
                              G_out, need > 0 ? ws : nullptr, (cudaStream_t)stream, 1);
}

int mlg_attention_stack(const mlg_csr* csr, int64_t n_centres, int32_t nnei_max,
                        int32_t channels, int32_t heads, int32_t n_layers, mlg_dtype dtype,
                        const void* const* W, const void* G_in, void* G_out, void* ws,
                        size_t ws_bytes, mlg_stream_t stream) {
  if (csr == nullptr) return MLG_ERR_INVALID_ARG;
  size_t need = mlg_attention_stack_workspace_bytes(csr->capacity, channels, n_layers, dtype);
  if (need > 0 && (ws == nullptr || ws_bytes < need)) return MLG_ERR_WORKSPACE;
  return attention_stack_impl(csr, n_centres, nnei_max, channels, heads, dtype, n_layers, W, G_in,
                              G_out, need > 0 ? ws : nullptr, (cudaStream_t)stream);
}

size_t mlg_forward_workspace_bytes(int64_t n_atoms, double rcut, const double box[9],
                                   const uint8_t pbc[3], int64_t capacity, int32_t channels,
                                   int32_t n_layers, mlg_dtype dtype) {
  size_t b = mlg_build_csr_workspace_bytes(n_atoms, rcut, box, pbc);
  if (b == 0 || capacity < 0 || channels < 1 || n_layers < 1) return 0;
  size_t el = dtype == MLG_F64 ? 8 : 4;
  if (n_layers >= 2) b = align_up(b) + align_up((size_t)capacity * channels * el);
  return b;
}

int mlg_forward(const mlg_system* sys, double rcut, double r_on, int32_t nnei_max,
                int32_t channels, int32_t heads, int32_t n_layers, mlg_dtype dtype,
                const void* const* W, const void* G0, void* G_out, const mlg_csr* csr,
                void* ws, size_t ws_bytes, mlg_stream_t stream) {
  if (sys == nullptr || W == nullptr || G0 == nullptr || G_out == nullptr || n_layers < 1)
    return MLG_ERR_INVALID_ARG;
  if (G0 == G_out) return MLG_ERR_INVALID_ARG;
  if (csr == nullptr) return MLG_ERR_INVALID_ARG;
  size_t need = mlg_forward_workspace_bytes(sys->n_atoms, rcut, sys->box, sys->pbc,
                                            csr->capacity, channels, n_layers, dtype);
  size_t build_need = mlg_build_csr_workspace_bytes(sys->n_atoms, rcut, sys->box, sys->pbc);
  if (need == 0 || build_need == 0) {
    // let the build report the precise argument error
    int rc = build_impl(sys, rcut, r_on, nnei_max, csr, nullptr, 0, (cudaStream_t)stream);
    return rc == MLG_OK ? MLG_ERR_INVALID_ARG : rc;
  }
  if (ws == nullptr || ws_bytes < need) return MLG_ERR_WORKSPACE;
  for (int k = 0; k < 3 * n_layers; ++k)
    if (W[k] == nullptr) return MLG_ERR_INVALID_ARG;
  int rc = build_impl(sys, rcut, r_on, nnei_max, csr, ws, build_need, (cudaStream_t)stream);
  if (rc != MLG_OK) return rc;
  void* pong = n_layers >= 2 ? static_cast<char*>(ws) + align_up(build_need) : nullptr;
  return attention_stack_impl(csr, sys->n_atoms, nnei_max, channels, heads, dtype, n_layers, W,
                              G0, G_out, pong, (cudaStream_t)stream);
}

int mlg_forward_launch_count(int64_t n_atoms, double rcut, const double box[9],
                             const uint8_t pbc[3], int32_t nnei_max, int32_t channels,
                             int32_t heads, int32_t n_layers, mlg_dtype dtype) {
  BuildPlan plan;
  if (n_layers < 1 || make_plan(n_atoms, rcut, box, pbc, &plan) != MLG_OK) return 0;
  auto scan_launches = [](int64_t n) { return n <= kScanSingleMax ? 1 : 3; };
  const int attn = forward_launches(n_atoms, nnei_max, channels, heads, n_layers, dtype);
  // one-launch build, or init, [bbox], bin, scan(cells), scatter, count,
  // scan(row_ptr), fill; then the attention
  if (use_fused_build(plan, n_atoms)) return 1 + attn;
  return 5 + (plan.any_open ? 1 : 0) + scan_launches(plan.ncell_cap) + scan_launches(n_atoms) +
         attn;
}

const char* mlg_attention_kernels(int32_t nnei_max, int32_t channels, int32_t heads,
                                  int32_t n_layers, mlg_dtype dtype) {
  if (channels < 1 || heads < 1 || channels % heads != 0 || n_layers < 1) return "";
  const int D = channels / heads;
  const int R = tile_rows(dtype, channels, D, nnei_max);
  if (R > 0 && n_layers <= kMaxFusedLayers) {
    if (dtype == MLG_F64) return nnei_max > R ? "k_attn_dmma + k_attn_generic" : "k_attn_dmma";
    if (kTcAttn && channels == 32 && D == 8 && n_layers == 1) {
#if MLG_TC_ATTN == 7
#define MLG_TC_NAME "k_attn_tc7 (tcgen05 logits, mma.sync P.V, rows <= 64)"
#elif MLG_TC_ATTN == 6
#define MLG_TC_NAME "k_attn_tc6 (tcgen05 logits, rows <= 64)"
#else
#define MLG_TC_NAME "k_attn_tc2 (tcgen05 logits and P.V, rows <= 64)"
#endif
      if (nnei_max > R) return MLG_TC_NAME " + k_attn_tc (rows <= 128) + k_attn_generic";
      if (nnei_max > tc2::MAXN) return MLG_TC_NAME " + k_attn_tc (rows <= 128)";
      return MLG_TC_NAME;
#undef MLG_TC_NAME
    }
    return nnei_max > R ? "k_attn_tc + k_attn_generic" : "k_attn_tc";
  }
  const int Rg = hg_rows(dtype, channels, D);
  if (Rg > 0) {
    const char* k = dtype == MLG_F32 ? "k_attn_hgtc" : "k_attn_hg";
    if (nnei_max <= Rg) return k;
    return dtype == MLG_F32 ? "k_attn_hgtc + k_attn_generic" : "k_attn_hg + k_attn_generic";
  }
  return "k_attn_generic";
}

const char* mlg_status_string(int status) {
  switch (status) {
    case MLG_OK: return "MLG_OK";
    case MLG_ERR_INVALID_ARG: return "MLG_ERR_INVALID_ARG: invalid argument";
    case MLG_ERR_WORKSPACE: return "MLG_ERR_WORKSPACE: workspace missing, too small or misaligned";
    case MLG_ERR_CAPACITY: return "MLG_ERR_CAPACITY: negative edge capacity";
    case MLG_ERR_INPUT_DATA: return "MLG_ERR_INPUT_DATA: invalid input data";
    case MLG_ERR_UNSUPPORTED: return "MLG_ERR_UNSUPPORTED: shape or cell not supported";
    case MLG_ERR_CUDA: return "MLG_ERR_CUDA: CUDA launch error";
    default: return "unknown mlg status";
  }
}

int mlg_exp2_neg(const double* y, double* out, int64_t n, mlg_stream_t stream) {
  if (n < 0 || (n > 0 && (y == nullptr || out == nullptr))) return MLG_ERR_INVALID_ARG;
  if (n == 0) return MLG_OK;
  const int64_t blocks = (n + 255) / 256;
  k_exp2_neg<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, (cudaStream_t)stream>>>(y, out,
                                                                                          n);
  return launch_status();
}

size_t mlg_verlet_workspace_bytes(int64_t n_atoms, double rcut, double skin, const double box[9],
                                  const uint8_t pbc[3]) {
  VerletLayout V;
  if (verlet_layout(n_atoms, rcut, skin, box, pbc, &V) != MLG_OK) return 0;
  return V.total;
}

int mlg_verlet_step(const mlg_system* sys, double rcut, double r_on, double skin,
                    int32_t nnei_max, const mlg_verlet_list* list, const mlg_csr* out, void* ws,
                    size_t ws_bytes, mlg_stream_t stream) {
  return verlet_step_impl(sys, rcut, r_on, skin, nnei_max, list, out, ws, ws_bytes,
                          (cudaStream_t)stream);
}

int mlg_build_csr_wait_test(const mlg_system* sys, double rcut, double r_on, int32_t nnei_max,
                             const mlg_csr* csr, void* ws, size_t ws_bytes, int32_t polls,
                             mlg_stream_t stream) {
  if (polls < 1) return MLG_ERR_INVALID_ARG;
  BuildOptions opt;
  opt.wait_test = true;
  opt.polls = polls;
  opt.hold_release = 1;
  return build_impl(sys, rcut, r_on, nnei_max, csr, ws, ws_bytes, (cudaStream_t)stream, opt);
}

int mlg_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free CSR build.
//
// For callers that cannot allocate device memory themselves: a force
// callback inside an MD engine that hands the library raw device pointers
// but owns every allocation (and must not stall its time step on the
// device-wide synchronisation an allocation can cause), or a host plugin
// that has no allocator of its own.  This entry point takes its scratch
// from a fixed array in the library's own device memory instead of a
// caller workspace.  It runs exactly the same kernels as mlg_build_csr.
#include <mutex>

namespace {

constexpr size_t kNoAllocScratchBytes = MLG_NOALLOC_SCRATCH_BYTES;

// One array per GPU that loads this library, held until the process exits.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices];  // device address of the array, per device
CUcontext g_noalloc_ctx[kNoAllocMaxDevices];  // the context that address belongs to

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// The calling thread's current context (nullptr if it cannot be read).
CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr)
      return nullptr;
    fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  CUcontext ctx = nullptr;
  return fn(&ctx) == CUDA_SUCCESS ? ctx : nullptr;
}

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with that device current and cached together with the context it belongs
// to; a new context of the device (after a device reset the module is loaded
// again, at a possibly different address) triggers a fresh lookup.
int noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MLG_ERR_CUDA;
  }
  if (dev < 0 || dev >= kNoAllocMaxDevices) return MLG_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  CUcontext ctx = current_context();
  if (g_noalloc_ptr[dev] == nullptr || ctx == nullptr || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return MLG_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = current_context();  // made current by the lookup if it was not yet
  }
  *out = g_noalloc_ptr[dev];
  return MLG_OK;
}

}  // namespace

extern "C" int mlg_build_csr_noalloc(const mlg_system* sys, double rcut, double r_on,
                                     int32_t nnei_max, const mlg_csr* csr,
                                     mlg_stream_t stream) {
  if (sys == nullptr) return MLG_ERR_INVALID_ARG;
  // what the build cannot do without (the array holds no key stash for
  // systems this size; the fill then searches the stencil again)
  size_t need = 0;
  {
    BuildPlan plan;
    if (make_plan(sys->n_atoms, rcut, sys->box, sys->pbc, &plan) == MLG_OK)
      need = build_layout(sys->n_atoms, plan.ncell_cap).total;
  }
  if (need == 0)  // invalid arguments: let the regular checks name the error
    return build_impl(sys, rcut, r_on, nnei_max, csr, nullptr, 0, (cudaStream_t)stream);
  if (need > kNoAllocScratchBytes) return MLG_ERR_WORKSPACE;  // system too large for the array
  void* scratch = nullptr;
  int rc = noalloc_scratch(&scratch);
  if (rc != MLG_OK) return rc;
  return build_impl(sys, rcut, r_on, nnei_max, csr, scratch, kNoAllocScratchBytes,
                    (cudaStream_t)stream);
}
