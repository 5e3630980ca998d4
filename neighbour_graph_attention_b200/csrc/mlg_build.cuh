// mlg_build.cuh -- stage 1: on-device destination CSR of all periodic
// neighbour images within rcut (sm_100a).
//
// What is built: the per-pair edge index / edge vector tensors of
// createEdgeTensors() (deepmd-kit issue "DPA4 .pt2 LAMMPS (C++ AOTI) inference
// 3-6x slower than Python (ASE)", Root cause analysis, bottleneck 1), emitted
// directly as the destination CSR (issue "NeighborGraph attention is 4-9x
// slower than dense", Proposed fix: destination_order / destination_row_ptr),
// with the per-centre cap sel (DPA4 issue, Reproduction: sel=181).  The
// search is the O(N) GPU cell list the DPA4 issue's Python path uses
// (Root cause analysis: "GPU O(N) cell list"), in the count -> prefix scan ->
// fill shape of its build_nlist_gpu() remark, rebuilt for sm_100a:
//
//   k_init     zero the cell histogram, counters and status
//   k_bbox     (open axes only) bounding box of the finite coordinates
//   k_bin      cell of each atom (wrapped into the box along periodic axes)
//              and its rank inside the cell from a warp-aggregated atomic
//   scan       exclusive scan of the histogram -> cell_start
//   k_scatter  atom records (coords, index, wrap image) in cell order
//   k_count    warp per destination: candidates of the stencil cells, exact
//              fp64 test r^2 < rcut^2, count -> kept = min(count, nnei_max)
//   scan       exclusive scan of kept -> row_ptr, E
//   k_fill     warp per destination: collect accepted candidates in shared
//              memory, select the nnei_max nearest when the row overflows,
//              sort into canonical (source, shift) order, write SoA edges
//
// Bit-exactness: the vector, distance and switch of an edge are computed with
// explicitly rounded operations (__dadd_rn, __dmul_rn, __dsqrt_rn, ...) in the
// one order that defines them, so no contraction into FMA can change a bit.
#pragma once

#include "mlg_common.cuh"

namespace mlg {

// ------------------------------------------------------------------ types

// An atom in cell order: original coordinates, index and packed wrap image
// (10 bits per axis, bias 512).
struct __align__(16) Rec {
  double x, y, z;
  int j;
  int w;
};

__host__ __device__ __forceinline__ int pack_w(int w0, int w1, int w2) {
  return (w0 + 512) | ((w1 + 512) << 10) | ((w2 + 512) << 20);
}
__device__ __forceinline__ int unpack_w(int p, int k) { return ((p >> (10 * k)) & 1023) - 512; }

// The cell grid as the device uses it.
struct CellGrid {
  double lo[3];     // grid origin along open axes (0 along periodic axes)
  double inv_h[3];  // cells per Angstrom (0 when an open axis has one cell)
  double L[3];      // box length along periodic axes
  double invL[3];
  int n[3];         // cells per axis
  int D[3];         // stencil reach in cells
  int periodic[3];
  int ncell;
  float Lf[3];      // box lengths as float (0 along open axes)
  float r2lo, r2hi; // fp32 prefilter: r2f < r2lo surely inside, r2f > r2hi surely outside
};

// What the host fixes before launch.
struct BuildPlan {
  int periodic[3];
  double L[3], invL[3], inv_h[3];
  int n_fixed[3];     // periodic axes: cells
  int D_fixed[3];     // periodic axes: stencil reach
  int n_open_max[3];  // open axes: most cells allowed
  double rcd;         // minimum cell size along open axes (rcut plus margin)
  double rc2;         // rcut * rcut
  int any_open;
  int ncell_cap;
  int max_reach;      // largest stencil reach over the axes
};

struct BuildArgs {
  int64_t n;
  const double* coords;
  const int32_t* types;
  int32_t n_types;
  double box[9];
  double rcut, r_on, rc2;
  int nnei_max;
  double taylor[12];  // Taylor coefficients (-1)^k / (2k+1)! of sin
  int64_t capacity;
  int64_t* row_ptr;
  int32_t* src;
  int32_t* shift;
  double* vec;
  double* dist;
  double* sw;
  int64_t* n_edges;
  int64_t* n_truncated;
  uint32_t* status;
  int32_t src_offset;        // added to written source indices (systems of a batch)
  int zero_globals;          // k_init clears n_truncated and status (not in a batch)
  long long spin_polls;      // one-launch build: polls of each bounded wait (0: the default)
  int hold_release;          // one-launch build: CTA 0 never releases the binned atoms, so
                             // the other CTAs' waits run out (tests of the timeout path)
  const uint32_t* gate;      // device word or nullptr: when it is 0 every kernel of the
                             // build returns at once (a rebuild decided on the device)
  // workspace
  CellGrid* grid;
  unsigned long long* bbox;  // [6] ordered bits: min x, y, z, max x, y, z
  int* cell_count;           // [ncell_cap + 1]
  int* cell_start;           // [ncell_cap + 1]
  int* atom_cell;            // [n]  (-1: left out)
  int* atom_rank;            // [n]
  int* atom_w;               // [n]
  Rec* recs;                 // [n]
  float4* pos4;              // [n] cell order: position in the grid frame (fp32), atom index
  int* kept;                 // [n]
  int* raw;                  // [n]
  long long* partial;        // scan partials
  unsigned long long* stash; // [n][kStashSlots] accepted keys of each row the count
                             // could keep whole (nullptr: none; the fill searches again)
  int* stash_n;              // [n] keys in the row's stash, -1: not stashed
  int stash_q;               // stash keys carry the source's cell-order record (n <= 2^21)
};

// False when the build is gated off by a device word (uniform for a launch:
// the word is written by an earlier kernel on the same stream).
__device__ __forceinline__ bool gated_off(const uint32_t* gate) {
  return gate != nullptr && *gate == 0u;
}

constexpr int kFillMaxCand = 256;  // shared-memory candidates per destination
// Rows of at most kStashSlots accepted candidates (and no truncation) keep
// their keys from the count to the fill, which then sorts and writes them
// without searching the stencil again.
constexpr int kStashSlots = 64;
constexpr int kCountWarps = 8;
constexpr int kFillWarps = 4;

// ------------------------------------------------------------- geometry

// r^2 of candidate (x_j + S L) - x_i.  Along a periodic (axis-aligned) axis the
// shift contributes S_k L_k; the other rows of the box contribute signed
// zeros only, which leave r^2 unchanged.
__device__ __forceinline__ double cand_r2(const CellGrid& g, const double* xi, const Rec& rc,
                                          const int* S) {
  double xj[3] = {rc.x, rc.y, rc.z};
  double v[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    double xs = g.periodic[k] ? __dadd_rn(xj[k], __dmul_rn((double)S[k], g.L[k])) : xj[k];
    v[k] = __dsub_rn(xs, xi[k]);
  }
  return __dadd_rn(__dadd_rn(__dmul_rn(v[0], v[0]), __dmul_rn(v[1], v[1])),
                   __dmul_rn(v[2], v[2]));
}

// The edge vector as defined for output:
//   sh_c = (S_0 a1_c + S_1 a2_c) + S_2 a3_c,  v_c = (x_j,c + sh_c) - x_i,c
__device__ __forceinline__ double edge_vec(const double* box, const double* xi,
                                           const double* xj, const int* S, double* v) {
  double s0 = (double)S[0], s1 = (double)S[1], s2 = (double)S[2];
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    double sh = __dadd_rn(__dmul_rn(s0, box[c]), __dmul_rn(s1, box[3 + c]));
    sh = __dadd_rn(sh, __dmul_rn(s2, box[6 + c]));
    v[c] = __dsub_rn(__dadd_rn(xj[c], sh), xi[c]);
  }
  return __dadd_rn(__dadd_rn(__dmul_rn(v[0], v[0]), __dmul_rn(v[1], v[1])),
                   __dmul_rn(v[2], v[2]));
}

// Cosine switch: 1 below r_on, 0 from rcut, else 0.5 (1 + cos(pi u)) with
// cos(pi u) = -sin(pi (u - 1/2)) and sin by its Taylor series through x^23
// (Horner in x^2).  Every operation explicitly rounded.
__device__ __forceinline__ double switch_fn(double r, double rcut, double r_on,
                                            const double* c) {
  if (r < r_on) return 1.0;
  if (r >= rcut) return 0.0;
  const double pi = 3.141592653589793;
  double u = __ddiv_rn(__dsub_rn(r, r_on), __dsub_rn(rcut, r_on));
  double x = __dmul_rn(pi, __dsub_rn(u, 0.5));
  double x2 = __dmul_rn(x, x);
  double p = c[11];
#pragma unroll
  for (int k = 10; k >= 0; --k) p = __dadd_rn(c[k], __dmul_rn(x2, p));
  double sinx = __dmul_rn(x, p);
  return __dmul_rn(0.5, __dadd_rn(1.0, -sinx));
}

// ------------------------------------------------------------ grid setup

__device__ __forceinline__ CellGrid derive_grid(const BuildPlan& p,
                                                const unsigned long long* bbox) {
  CellGrid g;
  int nc = 1;
  double ext = 0.0;  // largest coordinate span of the grid frame
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    g.periodic[k] = p.periodic[k];
    if (p.periodic[k]) {
      g.lo[k] = 0.0;
      g.L[k] = p.L[k];
      g.invL[k] = p.invL[k];
      g.inv_h[k] = p.inv_h[k];
      g.n[k] = p.n_fixed[k];
      g.D[k] = p.D_fixed[k];
    } else {
      g.L[k] = 0.0;
      g.invL[k] = 0.0;
      double lo = from_ordered_bits(bbox[k]);
      double hi = from_ordered_bits(bbox[3 + k]);
      int n = 1;
      double ext = hi - lo;
      if (lo <= hi && ext > 0.0) {
        double q = floor(ext / p.rcd);
        n = q < 1.0 ? 1 : (q > (double)p.n_open_max[k] ? p.n_open_max[k] : (int)q);
        while (n > 1 && ext / (double)n < p.rcd) --n;
      }
      g.lo[k] = lo <= hi ? lo : 0.0;
      if (lo <= hi) ext = fmax(ext, hi - lo);
      g.n[k] = n;
      g.inv_h[k] = n > 1 ? (double)n / ext : 0.0;
      g.D[k] = n > 1 ? 1 : 0;
    }
    nc *= g.n[k];
  }
  g.ncell = nc;
  // fp32 prefilter margin.  Positions are stored in the grid frame (wrapped
  // along periodic axes, shifted by the bounding-box origin along open ones),
  // |p| <= ext; an image adds +-L.  Each fp32 coordinate of a difference
  // carries at most 4 roundings of 2^-24 * 2 ext, so |delta_k| <= 2^-20 * ext
  // bounds its error with room to spare; r^2 then moves by at most
  // 2 sqrt(3) rcut delta + 3 delta^2 plus the fp32 rounding of the sum.
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    if (g.periodic[k]) ext = fmax(ext, g.L[k]);
    g.Lf[k] = (float)g.L[k];
  }
  const double rc = p.rcd, rc2 = rc * rc;
  const double dlt = 2.0 * 9.5367431640625e-07 * (ext + rc);  // 2 * 2^-20 * (ext + rc)
  const double margin = 2.0 * (3.4641016151377544 * rc * dlt + 3.0 * dlt * dlt) +
                        16.0 * 5.9604644775390625e-08 * rc2;
  g.r2lo = __double2float_rd(fmax(0.0, p.rc2 - margin));
  g.r2hi = __double2float_ru(p.rc2 + margin);
  return g;
}

// ----------------------------------------------------------------- kernels

__global__ void k_init(BuildArgs a, int ncell_cap) {
  if (gated_off(a.gate)) return;
  int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t m = t; m <= ncell_cap; m += stride) a.cell_count[m] = 0;
  if (t < 3) {
    a.bbox[t] = ~0ull;
    a.bbox[3 + t] = 0ull;
  }
  if (t == 0 && a.zero_globals) {
    *a.n_truncated = 0;
    *a.status = 0u;
  }
}

// Bounding box of the finite coordinates along open axes: atoms i0, i0 +
// stride, ... of this thread, folded into a.bbox (warp-collective).
__device__ void bbox_accumulate(const BuildArgs& a, const BuildPlan& p, int64_t i0,
                                int64_t stride) {
  double lo[3] = {INFINITY, INFINITY, INFINITY}, hi[3] = {-INFINITY, -INFINITY, -INFINITY};
  for (int64_t i = i0; i < a.n; i += stride) {
    double x0 = a.coords[3 * i], x1 = a.coords[3 * i + 1], x2 = a.coords[3 * i + 2];
    if (!(isfinite(x0) && isfinite(x1) && isfinite(x2))) continue;
    double x[3] = {x0, x1, x2};
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      lo[k] = fmin(lo[k], x[k]);
      hi[k] = fmax(hi[k], x[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    if (p.periodic[k]) continue;
    double l = lo[k], h = hi[k];
    for (int o = 16; o > 0; o >>= 1) {
      l = fmin(l, __shfl_xor_sync(kFull, l, o));
      h = fmax(h, __shfl_xor_sync(kFull, h, o));
    }
    if (lane_id() == 0 && l <= h) {
      atomicMin(&a.bbox[k], ordered_bits(l));
      atomicMax(&a.bbox[3 + k], ordered_bits(h));
    }
  }
}

__global__ void k_bbox(BuildArgs a, BuildPlan p) {
  if (gated_off(a.gate)) return;
  bbox_accumulate(a, p, (int64_t)blockIdx.x * blockDim.x + threadIdx.x,
                  (int64_t)gridDim.x * blockDim.x);
}

// Cell, wrap image and in-cell rank of atom i (i >= n: none), counted in the
// histogram `hist` (global or shared) with the rank in rank_out[i].  With
// s_cell / s_w the cell and image also go to those (shared) arrays.  Called
// by every lane of a warp (warp-aggregated histogram atomics).
__device__ __forceinline__ void bin_atom(const BuildArgs& a, const CellGrid& g, int64_t i,
                                         int* hist, int* rank_out, int* s_cell = nullptr,
                                         int* s_w = nullptr) {
  int cell = -1;
  uint32_t st = 0;
  if (i < a.n) {
    double x[3] = {a.coords[3 * i], a.coords[3 * i + 1], a.coords[3 * i + 2]};
    int wpack = 0;
    if (!(isfinite(x[0]) && isfinite(x[1]) && isfinite(x[2]))) {
      st |= MLG_STATUS_NONFINITE_COORD;
    } else {
      int c[3], w[3];
      bool ok = true;
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        double y;
        if (g.periodic[k]) {
          double fq = floor(x[k] * g.invL[k]);
          if (!(fabs(fq) <= 511.0)) {
            ok = false;
            fq = 0.0;
          }
          w[k] = (int)fq;
          y = x[k] - fq * g.L[k];
        } else {
          w[k] = 0;
          y = x[k] - g.lo[k];
        }
        double cf = floor(y * g.inv_h[k]);
        int ck = cf < 0.0 ? 0 : (cf >= (double)g.n[k] ? g.n[k] - 1 : (int)cf);
        c[k] = ck;
      }
      if (!ok) {
        st |= MLG_STATUS_IMAGE_RANGE;
      } else {
        cell = (c[0] * g.n[1] + c[1]) * g.n[2] + c[2];
        wpack = pack_w(w[0], w[1], w[2]);
      }
    }
    if (a.types != nullptr) {
      int t = a.types[i];
      if (t < 0 || t >= a.n_types) st |= MLG_STATUS_TYPE_RANGE;
    }
    a.atom_cell[i] = cell;
    a.atom_w[i] = wpack;
    if (s_cell != nullptr) {
      s_cell[i] = cell;
      s_w[i] = wpack;
    }
    if (cell < 0) {  // left out of the cell lists: no centre scan will visit it
      a.kept[i] = 0;
      a.raw[i] = 0;
    }
  }
  // warp-aggregated atomics on the cell histogram
  unsigned act = __ballot_sync(kFull, cell >= 0);
  if (cell >= 0) {
    unsigned peers = __match_any_sync(act, cell);
    int leader = __ffs(peers) - 1;
    int base = 0;
    if ((int)lane_id() == leader) base = atomicAdd(&hist[cell], __popc(peers));
    base = __shfl_sync(peers, base, leader);
    rank_out[i] = base + __popc(peers & lanemask_lt());
  }
  st = __reduce_or_sync(kFull, st);
  if (lane_id() == 0 && st) atomicOr(a.status, st);
}

__global__ void k_bin(BuildArgs a, BuildPlan p) {
  if (gated_off(a.gate)) return;
  CellGrid g = derive_grid(p, a.bbox);
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.grid = g;
  bin_atom(a, g, (int64_t)blockIdx.x * blockDim.x + threadIdx.x, a.cell_count, a.atom_rank);
}

// Record and fp32 position of atom i (wrap image wpack) at cell-order slot pos.
__device__ __forceinline__ void scatter_atom_at(const BuildArgs& a, const CellGrid& sg, int64_t i,
                                                int pos, int wpack) {
  Rec r;
  r.x = a.coords[3 * i];
  r.y = a.coords[3 * i + 1];
  r.z = a.coords[3 * i + 2];
  r.j = (int)i;
  r.w = wpack;
  a.recs[pos] = r;
  double x[3] = {r.x, r.y, r.z};
  float y[3];
#pragma unroll
  for (int k = 0; k < 3; ++k)
    y[k] = (float)(sg.periodic[k] ? x[k] - (double)unpack_w(r.w, k) * sg.L[k] : x[k] - sg.lo[k]);
  a.pos4[pos] = make_float4(y[0], y[1], y[2], __int_as_float((int)i));
}

__global__ void k_scatter(BuildArgs a) {
  if (gated_off(a.gate)) return;
  __shared__ CellGrid sg;
  if (threadIdx.x == 0) sg = *a.grid;
  __syncthreads();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.n) return;
  const int cell = a.atom_cell[i];
  if (cell < 0) return;
  scatter_atom_at(a, sg, i, a.cell_start[cell] + a.atom_rank[i], a.atom_w[i]);
}

// ----------------------------------------------------- candidate traversal

struct WarpScratch {
  int pre[33];
  int start[32];
  int tpack[32];
};

struct Centre {
  double x[3];
  int w[3];
  int c[3];
  int i;
};

__device__ __forceinline__ Centre load_centre(const BuildArgs& a, const CellGrid& g, int i,
                                              int cell) {
  Centre cc;
  cc.i = i;
  cc.x[0] = a.coords[3 * (int64_t)i];
  cc.x[1] = a.coords[3 * (int64_t)i + 1];
  cc.x[2] = a.coords[3 * (int64_t)i + 2];
  int wp = a.atom_w[i];
#pragma unroll
  for (int k = 0; k < 3; ++k) cc.w[k] = unpack_w(wp, k);
  cc.c[2] = cell % g.n[2];
  cc.c[1] = (cell / g.n[2]) % g.n[1];
  cc.c[0] = cell / (g.n[2] * g.n[1]);
  return cc;
}

// Visit every atom of the stencil cells of `cc` with its extended-cell image
// T.  The stencil cells are taken 32 at a time; their atom ranges are
// flattened with a warp prefix sum so that all lanes stay busy.  `f(valid,
// rec, tpack)` is called by all 32 lanes together (it may use warp votes).
template <class F>
__device__ __forceinline__ void for_each_candidate(const CellGrid& g, const int* cell_start,
                                                   const Centre& cc, WarpScratch& ws, F&& f) {
  const int lane = lane_id();
  const int w0 = 2 * g.D[0] + 1, w1 = 2 * g.D[1] + 1, w2 = 2 * g.D[2] + 1;
  const int s3 = w0 * w1 * w2;
  for (int chunk = 0; chunk < s3; chunk += 32) {
    int s = chunk + lane;
    int len = 0, start = 0, tp = 0;
    if (s < s3) {
      int d[3];
      d[2] = s % w2 - g.D[2];
      int t = s / w2;
      d[1] = t % w1 - g.D[1];
      d[0] = t / w1 - g.D[0];
      int m[3], T[3];
      bool ok = true;
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        int e = cc.c[k] + d[k];
        if (g.periodic[k]) {
          T[k] = floordiv(e, g.n[k]);
          m[k] = e - T[k] * g.n[k];
        } else {
          ok = ok && e >= 0 && e < g.n[k];
          m[k] = e;
          T[k] = 0;
        }
      }
      if (ok) {
        int cell = (m[0] * g.n[1] + m[1]) * g.n[2] + m[2];
        start = cell_start[cell];
        len = cell_start[cell + 1] - start;
        tp = ((T[0] + 64) << 14) | ((T[1] + 64) << 7) | (T[2] + 64);
      }
    }
    int incl = warp_incl_scan(len);
    int total = __shfl_sync(kFull, incl, 31);
    ws.pre[lane] = incl - len;
    ws.start[lane] = start;
    ws.tpack[lane] = tp;
    if (lane == 31) ws.pre[32] = total;
    __syncwarp();
    int o = 0;
    for (int base = 0; base < total; base += 32) {
      int t = base + lane;
      bool valid = t < total;
      int r = 0, tpo = 0;
      if (valid) {
        while (ws.pre[o + 1] <= t) ++o;
        r = ws.start[o] + (t - ws.pre[o]);
        tpo = ws.tpack[o];
      }
      f(valid, r, tpo);
    }
    __syncwarp();
  }
}

// Exact test of one candidate; returns true if (j, S) is an edge of cc.
__device__ __forceinline__ bool test_candidate(const CellGrid& g, const Centre& cc,
                                               const Rec& rc, int tpack, double rc2,
                                               double* r2_out) {
  int S[3];
  S[0] = ((tpack >> 14) & 127) - 64 + cc.w[0] - unpack_w(rc.w, 0);
  S[1] = ((tpack >> 7) & 127) - 64 + cc.w[1] - unpack_w(rc.w, 1);
  S[2] = (tpack & 127) - 64 + cc.w[2] - unpack_w(rc.w, 2);
  double r2 = cand_r2(g, cc.x, rc, S);
  *r2_out = r2;
  bool self = rc.j == cc.i && S[0] == 0 && S[1] == 0 && S[2] == 0;
  return r2 < rc2 && !self;
}

__global__ void __launch_bounds__(kCountWarps * 32) k_count(BuildArgs a) {
  if (gated_off(a.gate)) return;
  __shared__ CellGrid sg;
  __shared__ WarpScratch sw[kCountWarps];
  __shared__ int s_trunc;
  if (threadIdx.x == 0) {
    sg = *a.grid;
    s_trunc = 0;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const int64_t i = (int64_t)blockIdx.x * kCountWarps + warp;
  if (i < a.n) {
    int cell = a.atom_cell[i];
    int cnt = 0;
    if (cell >= 0) {
      Centre cc = load_centre(a, sg, (int)i, cell);
      for_each_candidate(sg, a.cell_start, cc, sw[warp], [&](bool valid, int r, int tp) {
        if (valid) {
          double r2;
          cnt += test_candidate(sg, cc, a.recs[r], tp, a.rc2, &r2) ? 1 : 0;
        }
      });
      cnt = warp_sum(cnt);
    }
    if (lane_id() == 0) {
      a.raw[i] = cnt;
      a.kept[i] = cnt < a.nnei_max ? cnt : a.nnei_max;
      if (cnt > a.nnei_max) atomicAdd(&s_trunc, 1);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_trunc) atomicAdd((unsigned long long*)a.n_truncated,
                                             (unsigned long long)s_trunc);
}

// ------------------------------------------------------------ warp sorts

__device__ __forceinline__ int next_pow2(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

// Ascending bitonic sort of k[0..n) (n <= kFillMaxCand) by one warp.
__device__ void warp_sort_keys(unsigned long long* k, int n) {
  const int lane = lane_id();
  const int P = next_pow2(n);
  for (int t = n + lane; t < P; t += 32) k[t] = ~0ull;
  __syncwarp();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = lane; t < (P >> 1); t += 32) {
        int lo = ((t & ~(stride - 1)) << 1) | (t & (stride - 1));
        int hi = lo + stride;
        bool up = (lo & size) == 0;
        unsigned long long x = k[lo], y = k[hi];
        if ((x > y) == up) {
          k[lo] = y;
          k[hi] = x;
        }
      }
      __syncwarp();
    }
  }
}

// Ascending bitonic sort of (d[t], k[t]) pairs by (d, k).
__device__ void warp_sort_pairs(unsigned long long* d, unsigned long long* k, int n) {
  const int lane = lane_id();
  const int P = next_pow2(n);
  for (int t = n + lane; t < P; t += 32) {
    d[t] = ~0ull;
    k[t] = ~0ull;
  }
  __syncwarp();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = lane; t < (P >> 1); t += 32) {
        int lo = ((t & ~(stride - 1)) << 1) | (t & (stride - 1));
        int hi = lo + stride;
        bool up = (lo & size) == 0;
        unsigned long long dx = d[lo], dy = d[hi], kx = k[lo], ky = k[hi];
        bool gt = dx > dy || (dx == dy && kx > ky);
        if (gt == up) {
          d[lo] = dy;
          d[hi] = dx;
          k[lo] = ky;
          k[hi] = kx;
        }
      }
      __syncwarp();
    }
  }
}

// Bitonic sorts of up to 64 elements held in registers, two per lane
// (element e = 32 r + lane in register r); padding elements are ~0.
__device__ __forceinline__ bool pair_lt(unsigned long long da, unsigned long long ka,
                                        unsigned long long db, unsigned long long kb) {
  return da < db || (da == db && ka < kb);
}

// ascending by (d, k)
__device__ __forceinline__ void warp_sort64_pairs(unsigned long long& d0, unsigned long long& k0,
                                                  unsigned long long& d1, unsigned long long& k1) {
  const int lane = lane_id();
#pragma unroll
  for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride == 32) {  // partner in the other register; size 64: ascending
        if (pair_lt(d1, k1, d0, k0)) {
          const unsigned long long td = d0, tk = k0;
          d0 = d1;
          k0 = k1;
          d1 = td;
          k1 = tk;
        }
      } else {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          unsigned long long& d = r ? d1 : d0;
          unsigned long long& k = r ? k1 : k0;
          const unsigned long long dp = __shfl_xor_sync(kFull, d, stride);
          const unsigned long long kp = __shfl_xor_sync(kFull, k, stride);
          const bool asc = ((32 * r + lane) & size) == 0;
          const bool keep_min = ((lane & stride) == 0) == asc;  // lower element of an ascending pair
          if (keep_min == pair_lt(dp, kp, d, k)) {
            d = dp;
            k = kp;
          }
        }
      }
    }
  }
}

// ascending
__device__ __forceinline__ void warp_sort64_keys(unsigned long long& k0, unsigned long long& k1) {
  const int lane = lane_id();
#pragma unroll
  for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride == 32) {
        if (k1 < k0) {
          const unsigned long long tk = k0;
          k0 = k1;
          k1 = tk;
        }
      } else {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          unsigned long long& k = r ? k1 : k0;
          const unsigned long long kp = __shfl_xor_sync(kFull, k, stride);
          const bool asc = ((32 * r + lane) & size) == 0;
          const bool keep_min = ((lane & stride) == 0) == asc;
          if (keep_min == (kp < k)) k = kp;
        }
      }
    }
  }
}

// ------------------------------------------------------------------- fill

// Stash key of a system of at most 2^21 atoms: source, packed image and the
// source's cell-order record index (the order is that of edge_key: (j, image)
// pairs are unique in a row, and the record follows from j).
__device__ __forceinline__ unsigned long long stash_key(int j, int tpack, int q) {
  return ((unsigned long long)j << 42) | ((unsigned long long)tpack << 21) |
         (unsigned long long)q;
}

__device__ __forceinline__ unsigned long long edge_key(int j, int tpack) {
  return ((unsigned long long)(unsigned)j << 21) | (unsigned long long)tpack;
}

// Key of a candidate staged in shared memory: the same (source, image) order
// as edge_key, with the staging slot (< 2048) in the low 11 bits.
constexpr int kSlotBits = 11;
__device__ __forceinline__ unsigned long long staged_key(int j, int tpack, int slot) {
  return ((unsigned long long)(unsigned)j << (21 + kSlotBits)) |
         ((unsigned long long)tpack << kSlotBits) | (unsigned long long)slot;
}
__device__ __forceinline__ int staged_src(unsigned long long key) {
  return (int)(key >> (21 + kSlotBits));
}
__device__ __forceinline__ int staged_image(unsigned long long key) {
  return (int)((key >> kSlotBits) & 0x1fffffull);
}
__device__ __forceinline__ int staged_slot(unsigned long long key) {
  return (int)(key & ((1ull << kSlotBits) - 1));
}

// Selection for rows with more than kFillMaxCand candidates, without a
// candidate buffer: bisection over the bit pattern of r^2 (monotone for
// non-negative doubles) finds the nnei_max-th smallest distance; a second
// bisection over the key (source, image) orders the candidates at exactly that
// distance.  Each probe rescans the row's candidates.  Writes the n kept keys
// to keys[0..n) (any order) and returns how many it wrote.
__device__ int fill_overflow_select(const BuildArgs& a, const CellGrid& g, const Centre& cc,
                                    WarpScratch& ws, unsigned long long* keys, int n,
                                    uint32_t* st) {
  (void)st;
  // count of candidates with (r2 bits, key) <= (b2, bk) in lexicographic order
  auto count_le = [&](unsigned long long b2, unsigned long long bk) {
    int cnt = 0;
    for_each_candidate(g, a.cell_start, cc, ws, [&](bool valid, int r, int tp) {
      if (valid) {
        const Rec rc = a.recs[r];
        double r2;
        if (test_candidate(g, cc, rc, tp, a.rc2, &r2)) {
          const unsigned long long b = (unsigned long long)__double_as_longlong(r2);
          const unsigned long long k = edge_key(rc.j, tp);
          if (b < b2 || (b == b2 && k <= bk)) ++cnt;
        }
      }
    });
    return warp_sum(cnt);
  };
  unsigned long long lo = 0ull, hi = (unsigned long long)__double_as_longlong(a.rc2);
  while (lo < hi) {  // smallest distance bits t with count(r2 <= t) >= n
    const unsigned long long mid = lo + ((hi - lo) >> 1);
    if (count_le(mid, ~0ull) >= n) hi = mid; else lo = mid + 1;
  }
  const unsigned long long t2 = lo;
  unsigned long long klo = 0ull, khi = (1ull << 53) - 1;
  while (klo < khi) {  // smallest key kt with count((r2, key) <= (t2, kt)) >= n
    const unsigned long long mid = klo + ((khi - klo) >> 1);
    if (count_le(t2, mid) >= n) khi = mid; else klo = mid + 1;
  }
  const unsigned long long tk = klo;
  int pos = 0;
  for_each_candidate(g, a.cell_start, cc, ws, [&](bool valid, int r, int tp) {
    bool take = false;
    unsigned long long key = 0;
    if (valid) {
      const Rec rc = a.recs[r];
      double r2;
      if (test_candidate(g, cc, rc, tp, a.rc2, &r2)) {
        const unsigned long long b = (unsigned long long)__double_as_longlong(r2);
        key = edge_key(rc.j, tp);
        take = b < t2 || (b == t2 && key <= tk);
      }
    }
    const unsigned m = __ballot_sync(kFull, take);
    if (take) {
      const int q = pos + __popc(m & lanemask_lt());
      if (q < n) keys[q] = key;
    }
    pos += __popc(m);
  });
  __syncwarp();
  return pos < n ? pos : n;
}

// Writes edge p of centre cc for `key` (a staged_key() with srec, else an
// edge_key()).
__device__ __forceinline__ void write_edge(const BuildArgs& a, const Centre& cc,
                                           unsigned long long key, int64_t p, const Rec* srec,
                                           bool qkey = false) {
  int j, tp, wj;
  double xj[3];
  if (qkey) {   // stash_key(): the source's record (one 32-byte sector)
    j = (int)(key >> 42);
    tp = (int)((key >> 21) & 0x1fffffull);
    const Rec rc = a.recs[(int)(key & 0x1fffffull)];
    wj = rc.w;
    xj[0] = rc.x;
    xj[1] = rc.y;
    xj[2] = rc.z;
  } else if (srec != nullptr) {
    j = staged_src(key);
    tp = staged_image(key);
    const Rec& rc = srec[staged_slot(key)];
    wj = rc.w;
    xj[0] = rc.x;
    xj[1] = rc.y;
    xj[2] = rc.z;
  } else {
    j = (int)(key >> 21);
    if (j < 0 || (int64_t)j >= a.n) return;
    tp = (int)(key & 0x1fffffull);
    wj = a.atom_w[j];
    xj[0] = a.coords[3 * (int64_t)j];
    xj[1] = a.coords[3 * (int64_t)j + 1];
    xj[2] = a.coords[3 * (int64_t)j + 2];
  }
  int S[3];
  S[0] = ((tp >> 14) & 127) - 64 + cc.w[0] - unpack_w(wj, 0);
  S[1] = ((tp >> 7) & 127) - 64 + cc.w[1] - unpack_w(wj, 1);
  S[2] = (tp & 127) - 64 + cc.w[2] - unpack_w(wj, 2);
  double v[3];
  double r2 = edge_vec(a.box, cc.x, xj, S, v);
  double r = __dsqrt_rn(r2);
  if (p < a.capacity) {
    a.src[p] = j + a.src_offset;
    a.shift[3 * p] = S[0];
    a.shift[3 * p + 1] = S[1];
    a.shift[3 * p + 2] = S[2];
    a.vec[3 * p] = v[0];
    a.vec[3 * p + 1] = v[1];
    a.vec[3 * p + 2] = v[2];
    a.dist[p] = r;
    a.sw[p] = switch_fn(r, a.rcut, a.r_on, a.taylor);
  }
}

// Sort the collected keys of one row into canonical order and write its
// edges.  keys/d2 hold m collected candidates (keys and exact r^2 bits, the
// latter needed when m > n); the row keeps n = min(raw, nnei_max): the n
// smallest by (r^2 bits, key), in key order.  With `srec`, the keys are
// staged_key()s and the source records come from srec; otherwise
// edge_key()s and global memory.  Rows of at most 64 candidates sort in
// registers.  Returns status bits.
__device__ uint32_t finish_row(const BuildArgs& a, const Centre& cc, unsigned long long* keys,
                               unsigned long long* d2, int n, int m, int64_t p0,
                               const Rec* srec = nullptr, bool qkey = false) {
  const int lane = lane_id();
  uint32_t st = 0;
  if (m > kFillMaxCand) m = kFillMaxCand;
  const int nv = n < m ? n : m;
  if (nv != n) st |= MLG_STATUS_INTERNAL;
  if (m <= 64) {
    unsigned long long k0 = lane < m ? keys[lane] : ~0ull;
    unsigned long long k1 = lane + 32 < m ? keys[lane + 32] : ~0ull;
    if (m > n) {
      unsigned long long e0 = lane < m ? d2[lane] : ~0ull;
      unsigned long long e1 = lane + 32 < m ? d2[lane + 32] : ~0ull;
      warp_sort64_pairs(e0, k0, e1, k1);
      if (lane >= nv) k0 = ~0ull;
      if (lane + 32 >= nv) k1 = ~0ull;
    }
    warp_sort64_keys(k0, k1);
    if (lane < nv) write_edge(a, cc, k0, p0 + lane, srec, qkey);
    if (lane + 32 < nv) write_edge(a, cc, k1, p0 + lane + 32, srec, qkey);
    return st;
  }
  if (m > n) warp_sort_pairs(d2, keys, m);
  warp_sort_keys(keys, nv);
  for (int e = lane; e < nv; e += 32) write_edge(a, cc, keys[e], p0 + e, srec, qkey);
  return st;
}

// One row from the global cell lists (rows beyond the shared-memory
// candidate capacity take the threshold search).
__device__ uint32_t fill_row_global(const BuildArgs& a, const CellGrid& g, const Centre& cc,
                                    WarpScratch& ws, unsigned long long* keys,
                                    unsigned long long* d2, int n, int raw, int64_t p0) {
  uint32_t st = 0;
  if (raw <= kFillMaxCand) {
    int pos = 0;
    for_each_candidate(g, a.cell_start, cc, ws, [&](bool valid, int r, int tp) {
      bool acc = false;
      unsigned long long key = 0, b = 0;
      if (valid) {
        const Rec rc = a.recs[r];
        double r2;
        acc = test_candidate(g, cc, rc, tp, a.rc2, &r2);
        key = edge_key(rc.j, tp);
        b = (unsigned long long)__double_as_longlong(r2);
      }
      unsigned m = __ballot_sync(kFull, acc);
      if (acc) {
        int q = pos + __popc(m & lanemask_lt());
        if (q < kFillMaxCand) {
          keys[q] = key;
          d2[q] = b;
        }
      }
      pos += __popc(m);
    });
    __syncwarp();
    st |= finish_row(a, cc, keys, d2, n, pos, p0);
  } else {
    const int nv = fill_overflow_select(a, g, cc, ws, keys, n, &st);
    st |= finish_row(a, cc, keys, d2, nv, nv, p0);
    if (nv != n) st |= MLG_STATUS_INTERNAL;
  }
  return st;
}

__global__ void __launch_bounds__(kFillWarps * 32) k_fill(BuildArgs a) {
  if (gated_off(a.gate)) return;
  __shared__ CellGrid sg;
  __shared__ WarpScratch sws[kFillWarps];
  extern __shared__ unsigned long long s_fill[];  // [warps][2][kFillMaxCand]
  if (threadIdx.x == 0) sg = *a.grid;
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const int64_t i = (int64_t)blockIdx.x * kFillWarps + warp;
  if (i >= a.n) return;
  const int cell = a.atom_cell[i];
  const int n = a.kept[i];
  if (cell < 0 || n == 0) return;
  unsigned long long* keys = s_fill + (size_t)warp * 2 * kFillMaxCand;
  Centre cc = load_centre(a, sg, (int)i, cell);
  uint32_t st = fill_row_global(a, sg, cc, sws[warp], keys, keys + kFillMaxCand, n, a.raw[i],
                                a.row_ptr[i]);
  if (lane_id() == 0 && st) atomicOr(a.status, st);
}

// ------------------------------------------------------------ per-cell scans
//
// One CTA per cell: every centre of a cell has the same 27 stencil cells, so
// their atoms are staged once in shared memory as fp32 positions with the
// image offset T L already added.  A candidate then costs one 16-byte
// shared load and a few fp32 operations; only candidates within the margin
// of rcut^2 (r2lo <= r2f <= r2hi) take the exact fp64 test, so the accept
// decision is the fp64 one bit for bit.  With REC the candidates' exact
// records are staged too, so the fp64 tests and the edge output read shared
// memory only.  Cells whose stencil holds more than kCellCand atoms fall back
// to the per-centre traversal of global memory.
constexpr int kCellCand = 768;       // stage capacity of the kernel chain
constexpr int kCellCandSmall = 2048; // one-launch build of systems of at most 75 atoms
constexpr int kCellWarps = 8;   // warps of the one-launch build's CTAs
// warps of the per-cell count and fill CTAs of the kernel chain, and their
// minimum resident CTAs per SM (launch bounds)
#ifndef MLG_SCAN_WARPS
#define MLG_SCAN_WARPS 8
#endif
#ifndef MLG_COUNT_MINB
#define MLG_COUNT_MINB 4
#endif
#ifndef MLG_FILL_MINB
#define MLG_FILL_MINB 4
#endif
constexpr int kScanWarps = MLG_SCAN_WARPS;
static_assert(kCellCandSmall <= (1 << kSlotBits), "staged_key slot bits");

template <int CAP>
struct CellStageT {
  int pre[33];      // candidate offset of each stencil cell
  int start[32];
  int tpack[32];
  int ncand;
  int fallback;
  int trunc;
  int staged_cell;          // cell whose candidates the arrays hold (-1: none)
  int self_pre;             // first slot of the cell's own (zero-image) stencil entry
  int c_lo, c_hi;           // the staged cell's centres (cell-order range)
  int stash_ci[kCellWarps];   // STASH: centre whose accepted keys a warp still holds (-1: none)
  int stash_cnt[kCellWarps];  // and how many
  float4 cand[CAP + 64];  // position + image offset, atom index in .w; padded with
                          // far-away sentinels to a multiple of 64 slots
  int cq[CAP];        // cell-order index (record of the exact data)
  int ct[CAP];        // packed image of the stencil cell
};
using CellStage = CellStageT<kCellCand>;

// Dynamic shared memory of the per-cell scans (NW warps): the stage, the
// fill's key buffers, and (REC) the candidates' exact records.
template <int CAP, int NW = kCellWarps>
struct CellSmem {
  static constexpr size_t keys_bytes = (size_t)NW * 2 * kFillMaxCand * sizeof(unsigned long long);
  static constexpr size_t keys_off = ((sizeof(CellStageT<CAP>) + 15) / 16) * 16;
  static constexpr size_t rec_off = keys_off + keys_bytes;
  static constexpr size_t bytes(bool fill, bool rec) {
    return rec ? rec_off + (size_t)CAP * sizeof(Rec) : keys_off + (fill ? keys_bytes : 0);
  }
};
__host__ __device__ constexpr size_t cellscan_smem(bool fill, bool rec = false) {
  return CellSmem<kCellCand, kScanWarps>::bytes(fill, rec);
}

// Count (FILL = false: raw, kept, truncations) or fill (FILL: the CSR rows)
// of the centres of `cell` taken by split `ys` of `nsplit` (centres
// c_lo + ys * kCellWarps + warp, stepping by nsplit * kCellWarps).  Called by
// every thread of the CTA.  Row starts come from row_off (tile-local copy of
// row_ptr, indexed by centre) or else from a.row_ptr.  Staged candidates of
// the same cell from an earlier call are reused.  With STASH (and REC) the
// count keeps each warp's accepted keys and distances in its key buffer, and
// a fill of the same centre by the same warp starts from them.
template <bool FILL, bool REC, bool STASH = false, int CAP = kCellCand, int NW = kCellWarps,
          bool GST = false>
__device__ void cellscan_item(const BuildArgs& a, const CellGrid& sg, WarpScratch* sws,
                              unsigned char* s_dyn, int cell, int ys, int nsplit,
                              const int* row_off) {
  CellStageT<CAP>& cs = *reinterpret_cast<CellStageT<CAP>*>(s_dyn);
  unsigned long long* s_keys =
      reinterpret_cast<unsigned long long*>(s_dyn + CellSmem<CAP, NW>::keys_off);
  Rec* s_rec = reinterpret_cast<Rec*>(s_dyn + CellSmem<CAP, NW>::rec_off);  // REC only
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (cell >= sg.ncell) return;
  const bool reuse = cs.staged_cell == cell;
  const int c_lo = reuse ? cs.c_lo : a.cell_start[cell];
  const int c_hi = reuse ? cs.c_hi : a.cell_start[cell + 1];
  if (c_lo + ys * NW >= c_hi) return;
  const int cz = cell % sg.n[2], cy = (cell / sg.n[2]) % sg.n[1], cx = cell / (sg.n[2] * sg.n[1]);
  // (GST fill) a row is stashed when the count kept all its accepted keys
  auto stashed = [&](int i) { return a.stash_n[i] >= 0; };
  if (GST && FILL) {
    // the stashed rows of this split's centres, straight from the count's
    // keys: sort and write; the stencil is staged only if a row is left
    unsigned long long* wkeys =
        reinterpret_cast<unsigned long long*>(s_dyn + CellSmem<CAP, NW>::keys_off) +
        (size_t)warp * 2 * kFillMaxCand;
    uint32_t st0 = 0;
    int left = 0;
    for (int ci = c_lo + ys * NW + warp; ci < c_hi; ci += nsplit * NW) {
      const Rec rci = a.recs[ci];
      const int i = rci.j;
      if (!stashed(i)) {
        left = 1;
        continue;
      }
      const int n = a.stash_n[i];
      if (n == 0) continue;
      for (int q = lane; q < n; q += 32) wkeys[q] = a.stash[(int64_t)i * kStashSlots + q];
      __syncwarp();
      Centre cc;
      cc.i = i;
      cc.x[0] = rci.x;
      cc.x[1] = rci.y;
      cc.x[2] = rci.z;
#pragma unroll
      for (int k = 0; k < 3; ++k) cc.w[k] = unpack_w(rci.w, k);
      cc.c[0] = cx;
      cc.c[1] = cy;
      cc.c[2] = cz;
      st0 |= finish_row(a, cc, wkeys, wkeys + kFillMaxCand, n, n, a.row_ptr[i], nullptr,
                        a.stash_q != 0);
      __syncwarp();
    }
    st0 = __reduce_or_sync(kFull, st0);
    if (lane == 0 && st0) atomicOr(a.status, st0);
    if (!__syncthreads_or(left)) return;
  }
  if (!reuse) {
    __syncthreads();  // earlier readers of the staging arrays are done
    if (warp == 0) {
      // stencil (reach <= 1 on every axis: at most 27 cells)
      const int w0 = 2 * sg.D[0] + 1, w1 = 2 * sg.D[1] + 1, w2 = 2 * sg.D[2] + 1;
      const int s3 = w0 * w1 * w2;
      int len = 0, start = 0, tp = 0;
      if (lane < s3) {
        int d[3];
        d[2] = lane % w2 - sg.D[2];
        d[1] = (lane / w2) % w1 - sg.D[1];
        d[0] = lane / (w2 * w1) - sg.D[0];
        const int c[3] = {cx, cy, cz};
        int m[3], T[3];
        bool ok = true;
#pragma unroll
        for (int k = 0; k < 3; ++k) {
          int e = c[k] + d[k];
          if (sg.periodic[k]) {
            T[k] = floordiv(e, sg.n[k]);
            m[k] = e - T[k] * sg.n[k];
          } else {
            ok = ok && e >= 0 && e < sg.n[k];
            m[k] = e;
            T[k] = 0;
          }
        }
        if (ok) {
          int cc = (m[0] * sg.n[1] + m[1]) * sg.n[2] + m[2];
          start = a.cell_start[cc];
          len = a.cell_start[cc + 1] - start;
          tp = ((T[0] + 64) << 14) | ((T[1] + 64) << 7) | (T[2] + 64);
        }
      }
      int incl = warp_incl_scan(len);
      cs.pre[lane] = incl - len;
      cs.start[lane] = start;
      cs.tpack[lane] = tp;
      if (lane == (sg.D[0] * w1 + sg.D[1]) * w2 + sg.D[2]) cs.self_pre = incl - len;
      if (lane == 31) {
        cs.pre[32] = incl;
        cs.ncand = incl;
        cs.fallback = incl > CAP;
        cs.trunc = 0;
        cs.staged_cell = cell;
        cs.c_lo = c_lo;
        cs.c_hi = c_hi;
      }
    }
    if (STASH && tid < NW) cs.stash_ci[tid] = -1;  // stashed slots refer to the old staging
    __syncthreads();
    if (!cs.fallback) {
      // stage the candidates: slot t of stencil cell s (pre[s] <= t <
      // pre[s + 1]); two slots per thread and round, loads first
      const int K = cs.ncand;
      constexpr int NT = NW * 32;
      for (int t0 = tid; t0 < K; t0 += 2 * NT) {
        int q[2], tp[2];
        float4 pv[2];
        Rec rv[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int t = t0 + u * NT;
          q[u] = -1;
          if (t < K) {
            int lo = 0, hi = 31;  // largest s with pre[s] <= t
            while (lo < hi) {
              const int mid = (lo + hi + 1) >> 1;
              if (cs.pre[mid] <= t) lo = mid; else hi = mid - 1;
            }
            q[u] = cs.start[lo] + (t - cs.pre[lo]);
            tp[u] = cs.tpack[lo];
            pv[u] = a.pos4[q[u]];
            if (REC) rv[u] = a.recs[q[u]];
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (q[u] < 0) continue;
          const int t = t0 + u * NT;
          float4 p = pv[u];
          p.x += (float)(((tp[u] >> 14) & 127) - 64) * sg.Lf[0];
          p.y += (float)(((tp[u] >> 7) & 127) - 64) * sg.Lf[1];
          p.z += (float)((tp[u] & 127) - 64) * sg.Lf[2];
          cs.cand[t] = p;
          cs.cq[t] = q[u];
          cs.ct[t] = tp[u];
          if (REC) s_rec[t] = rv[u];
        }
      }
      // sentinels up to a multiple of 64 slots: far away, so never accepted
      // and never near the cutoff (their squared distance overflows to +inf)
      for (int t = K + tid; t < ((K + 63) & ~63); t += NT)
        cs.cand[t] = make_float4(1e30f, 1e30f, 1e30f, __int_as_float(-1));
    }
    __syncthreads();
  } else if (!FILL && threadIdx.x == 0) {
    cs.trunc = 0;
  }
  if (!FILL) __syncthreads();
  const int K = cs.ncand;
  unsigned long long* keys = s_keys + (size_t)warp * 2 * kFillMaxCand;
  uint32_t st = 0;
  for (int ci = c_lo + ys * NW + warp; ci < c_hi; ci += nsplit * NW) {
    // the centre's own record: staged (self stencil cell) or global
    const int self_slot = cs.self_pre + (ci - c_lo);
    const bool staged_self = REC && !cs.fallback;
    const Rec rci = staged_self ? s_rec[self_slot] : a.recs[ci];
    const int i = rci.j;
    Centre cc;
    cc.i = i;
    cc.x[0] = rci.x;
    cc.x[1] = rci.y;
    cc.x[2] = rci.z;
#pragma unroll
    for (int k = 0; k < 3; ++k) cc.w[k] = unpack_w(rci.w, k);
    cc.c[0] = cx;
    cc.c[1] = cy;
    cc.c[2] = cz;
    const int64_t p0 = FILL ? (row_off != nullptr ? (int64_t)row_off[i] : a.row_ptr[i]) : 0;
    if (cs.fallback) {
      if (!FILL) {
        int cnt = 0;
        for_each_candidate(sg, a.cell_start, cc, sws[warp], [&](bool valid, int r, int tp) {
          if (valid) {
            double r2;
            cnt += test_candidate(sg, cc, a.recs[r], tp, a.rc2, &r2) ? 1 : 0;
          }
        });
        cnt = warp_sum(cnt);
        if (lane == 0) {
          a.raw[i] = cnt;
          a.kept[i] = cnt < a.nnei_max ? cnt : a.nnei_max;
          if (cnt > a.nnei_max) atomicAdd(&cs.trunc, 1);
          if (GST) a.stash_n[i] = -1;   // the fill searches again
        }
      } else {
        const int n = a.kept[i];
        if (n > 0)
          st |= fill_row_global(a, sg, cc, sws[warp], keys, keys + kFillMaxCand, n, a.raw[i], p0);
      }
      continue;
    }
    if (FILL && STASH && cs.stash_ci[warp] == ci) {
      // the count pass left this centre's accepted keys and distances here
      const int raw = cs.stash_cnt[warp];
      const int n = raw < a.nnei_max ? raw : a.nnei_max;
      if (n > 0) st |= finish_row(a, cc, keys, keys + kFillMaxCand, n, raw, p0, s_rec);
      continue;
    }
    if (GST && FILL && stashed(i)) continue;   // written from the stash above
    const int n = FILL ? a.kept[i] : 0;
    if (FILL && n == 0) continue;
    if (STASH) {
      __syncwarp();
      if (lane == 0) cs.stash_ci[warp] = -1;  // the key buffer is about to be overwritten
    }
    const float4 pi = staged_self ? cs.cand[self_slot] : a.pos4[ci];
    const bool need_d2 = FILL && a.raw[i] > n;
    constexpr bool kCollect = FILL || STASH;
    // (GST count) each lane's accepted candidates as bits: bit 2 s + u for slot
    // 64 s + lane + 32 u; the keys are formed once the row is known to fit
    constexpr bool kMask = GST && !FILL;
    uint32_t amask = 0;
    int cnt = 0;
    // the candidates, two per lane per step (slots t0 and t0 + 32 of a block
    // of 64); the fp32 prefilter decides all but the few within its margin of
    // rcut^2, which take the exact test outside the common path.  The centre
    // itself is the staged slot self_slot (its own cell, image 0).
    auto collect = [&](bool acc, int t, const float4& c) {
      const unsigned m = __ballot_sync(kFull, acc);
      if (acc) {
        const int qd = cnt + __popc(m & lanemask_lt());
        if (qd < kFillMaxCand) {
          const int j = __float_as_int(c.w), tp = cs.ct[t];
          keys[qd] = REC ? staged_key(j, tp, t) : edge_key(j, tp);
          if (!REC && need_d2) {
            double r2;
            test_candidate(sg, cc, a.recs[cs.cq[t]], tp, a.rc2, &r2);
            keys[kFillMaxCand + qd] = (unsigned long long)__double_as_longlong(r2);
          }
        }
      }
      cnt += __popc(m);
    };
    const int Kp = (K + 63) & ~63;
    for (int base = 0; base < Kp; base += 64) {
      const int t0 = base + lane, t1 = t0 + 32;
      const float4 c0 = cs.cand[t0], c1 = cs.cand[t1];
      const float dx0 = c0.x - pi.x, dy0 = c0.y - pi.y, dz0 = c0.z - pi.z;
      const float dx1 = c1.x - pi.x, dy1 = c1.y - pi.y, dz1 = c1.z - pi.z;
      const float r0 = fmaf(dz0, dz0, fmaf(dy0, dy0, dx0 * dx0));
      const float r1 = fmaf(dz1, dz1, fmaf(dy1, dy1, dx1 * dx1));
      bool a0 = r0 < sg.r2lo && t0 != self_slot;
      bool a1 = r1 < sg.r2lo && t1 != self_slot;
      const bool e0 = !(r0 < sg.r2lo) && r0 <= sg.r2hi;
      const bool e1 = !(r1 < sg.r2lo) && r1 <= sg.r2hi;
      if (__any_sync(kFull, e0 || e1)) {
        double r2;
        if (e0) a0 = test_candidate(sg, cc, REC ? s_rec[t0] : a.recs[cs.cq[t0]], cs.ct[t0],
                                    a.rc2, &r2);
        if (e1) a1 = test_candidate(sg, cc, REC ? s_rec[t1] : a.recs[cs.cq[t1]], cs.ct[t1],
                                    a.rc2, &r2);
      }
      if (!kCollect) {
        cnt += (a0 ? 1 : 0) + (a1 ? 1 : 0);
        if (kMask) amask |= ((a0 ? 1u : 0u) | (a1 ? 2u : 0u)) << (base >> 5);
      } else {
        collect(a0, t0, c0);
        collect(a1, t1, c1);
      }
    }
    if (REC && kCollect && (FILL ? need_d2 : cnt > a.nnei_max) && cnt <= kFillMaxCand) {
      // exact distances of a truncated row's accepted candidates, after the
      // scan (their slots are in the keys)
      __syncwarp();
      for (int q = lane; q < cnt; q += 32) {
        const unsigned long long key = keys[q];
        double r2;
        test_candidate(sg, cc, s_rec[staged_slot(key)], staged_image(key), a.rc2, &r2);
        keys[kFillMaxCand + q] = (unsigned long long)__double_as_longlong(r2);
      }
    }
    if (!FILL) {
      const int lane_cnt = cnt;
      if (!kCollect) cnt = warp_sum(cnt);  // collecting lanes hold the warp total already
      if (lane == 0) {
        a.raw[i] = cnt;
        a.kept[i] = cnt < a.nnei_max ? cnt : a.nnei_max;
        if (cnt > a.nnei_max) atomicAdd(&cs.trunc, 1);
        if (STASH && cnt <= kFillMaxCand) {
          cs.stash_ci[warp] = ci;
          cs.stash_cnt[warp] = cnt;
        }
      }
      if (GST) {
        // the row's keys for the fill (any order: the fill sorts them), each
        // lane's after the lanes below it
        const bool whole = cnt <= kStashSlots && cnt <= a.nnei_max;
        if (whole) {
          int q = lane_cnt;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(kFull, q, o);
            if (lane >= o) q += v;
          }
          q -= lane_cnt;   // exclusive
          unsigned long long* dst = a.stash + (int64_t)i * kStashSlots;
          for (uint32_t m = amask; m != 0; m &= m - 1) {
            const int b = __ffs(m) - 1;
            const int t = 32 * b + lane;   // slot 64 (b / 2) + 32 (b % 2) + lane
            const int j = __float_as_int(cs.cand[t].w);
            dst[q++] = a.stash_q ? stash_key(j, cs.ct[t], cs.cq[t]) : edge_key(j, cs.ct[t]);
          }
        }
        if (lane == 0) a.stash_n[i] = whole ? cnt : -1;
      }
    } else {
      __syncwarp();
      if (cnt > kFillMaxCand) {
        // more candidates than a warp holds: threshold search from global memory
        st |= fill_row_global(a, sg, cc, sws[warp], keys, keys + kFillMaxCand, n, cnt, p0);
      } else {
        st |= finish_row(a, cc, keys, keys + kFillMaxCand, n, cnt, p0, REC ? s_rec : nullptr);
      }
    }
  }
  if (FILL) {
    st = __reduce_or_sync(kFull, st);
    if (lane == 0 && st) atomicOr(a.status, st);
  } else {
    __syncthreads();
    if (tid == 0 && cs.trunc)
      atomicAdd((unsigned long long*)a.n_truncated, (unsigned long long)cs.trunc);
  }
}

template <bool FILL, bool GST = false>
__global__ void __launch_bounds__(kScanWarps * 32, FILL ? MLG_FILL_MINB : MLG_COUNT_MINB)
    k_cellscan(BuildArgs a) {
  if (gated_off(a.gate)) return;
  __shared__ CellGrid sg;
  __shared__ WarpScratch sws[kScanWarps];
  extern __shared__ __align__(16) unsigned char s_dyn[];
  if (threadIdx.x == 0) {
    sg = *a.grid;
    reinterpret_cast<CellStage*>(s_dyn)->staged_cell = -1;
  }
  __syncthreads();
  // blockIdx.y splits a cell's centres over several CTAs (small grids)
  cellscan_item<FILL, false, false, kCellCand, kScanWarps, GST>(a, sg, sws, s_dyn, blockIdx.x,
                                                                blockIdx.y, gridDim.y, nullptr);
}

// ------------------------------------------------------------------ scans
//
// Exclusive scan of int counts into int or int64 offsets: reduce-then-scan
// over tiles of 2048 (no inter-block waiting).  Small inputs use one block.

constexpr int kScanThreads = 256;
constexpr int kScanItems = 8;
constexpr int kScanTile = kScanThreads * kScanItems;
constexpr int kScanSingleMax = 1 << 13;

// exclusive block scan (blockDim.x threads, multiple of 32, <= 1024)
template <typename T>
__device__ __forceinline__ T block_excl_scan(T v, T* total) {
  __shared__ T s_w[33];
  const int lane = lane_id(), warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  T incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T u = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) s_w[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    T x = lane < nw ? s_w[lane] : T(0);
    T xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      T u = __shfl_up_sync(kFull, xi, o);
      if (lane >= o) xi += u;
    }
    if (lane < nw) s_w[lane] = xi - x;
    if (lane == 31) s_w[32] = xi;
  }
  __syncthreads();
  *total = s_w[32];
  T r = s_w[warp] + incl - v;
  __syncthreads();
  return r;
}

// Finishing of a row_ptr scan: E, capacity check.
struct ScanTail {
  int64_t* n_edges;
  uint32_t* status;
  int64_t capacity;
  const uint32_t* gate;  // as BuildArgs::gate (nullptr: always run)
};

// One block: tiles of blockDim.x x 4 items, each thread 4 contiguous items,
// carry from tile to tile.  Called by every thread of the block.
template <typename TOut>
__device__ void scan_block(const int* in, int64_t n, TOut* out, ScanTail tail) {
  long long carry = 0;
  for (int64_t base = 0; base < n; base += 4 * (int64_t)blockDim.x) {
    const int64_t t0 = base + 4 * (int64_t)threadIdx.x;
    int v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = t0 + u < n ? in[t0 + u] : 0;
    const long long s = (long long)v[0] + v[1] + v[2] + v[3];
    long long tot;
    long long off = block_excl_scan<long long>(s, &tot) + carry;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (t0 + u < n) out[t0 + u] = (TOut)off;
      off += v[u];
    }
    carry += tot;
  }
  if (threadIdx.x == 0) {
    out[n] = (TOut)carry;
    if (tail.n_edges) {
      *tail.n_edges = carry;
      if (carry > tail.capacity) atomicOr(tail.status, (uint32_t)MLG_STATUS_CAPACITY);
    }
  }
}

template <typename TOut>
__global__ void __launch_bounds__(1024) k_scan_single(const int* in, int64_t n, TOut* out,
                                                      ScanTail tail) {
  if (gated_off(tail.gate)) return;
  scan_block<TOut>(in, n, out, tail);
}

__global__ void __launch_bounds__(kScanThreads) k_scan_reduce(const int* in, int64_t n,
                                                              long long* partial,
                                                              const uint32_t* gate) {
  if (gated_off(gate)) return;
  const int64_t base = (int64_t)blockIdx.x * kScanTile;
  long long s = 0;
#pragma unroll
  for (int q = 0; q < kScanItems; ++q) {
    int64_t t = base + q * kScanThreads + threadIdx.x;
    if (t < n) s += in[t];
  }
  s = warp_sum(s);
  __shared__ long long s_w[kScanThreads / 32];
  if (lane_id() == 0) s_w[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long tot = 0;
    for (int w = 0; w < kScanThreads / 32; ++w) tot += s_w[w];
    partial[blockIdx.x] = tot;
  }
}

// one block: exclusive scan of the tile sums in place; partial[ntiles] = total
__global__ void __launch_bounds__(1024) k_scan_top(long long* partial, int ntiles,
                                                   const uint32_t* gate) {
  if (gated_off(gate)) return;
  long long carry = 0;
  for (int base = 0; base < ntiles; base += blockDim.x) {
    int t = base + threadIdx.x;
    long long v = t < ntiles ? partial[t] : 0;
    long long tot;
    long long ex = block_excl_scan<long long>(v, &tot);
    if (t < ntiles) partial[t] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) partial[ntiles] = carry;
}

template <typename TOut>
__global__ void __launch_bounds__(kScanThreads) k_scan_down(const int* in, int64_t n,
                                                            const long long* partial,
                                                            int ntiles, TOut* out,
                                                            ScanTail tail) {
  if (gated_off(tail.gate)) return;
  const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanItems;
  int v[kScanItems];
  long long s = 0;
#pragma unroll
  for (int q = 0; q < kScanItems; ++q) {
    int64_t t = base + q;
    v[q] = t < n ? in[t] : 0;
    s += v[q];
  }
  long long tot;
  long long off = block_excl_scan<long long>(s, &tot) + partial[blockIdx.x];
#pragma unroll
  for (int q = 0; q < kScanItems; ++q) {
    int64_t t = base + q;
    if (t < n) out[t] = (TOut)off;
    off += v[q];
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    long long total = partial[ntiles];
    out[n] = (TOut)total;
    if (tail.n_edges) {
      *tail.n_edges = total;
      if (total > tail.capacity) atomicOr(tail.status, (uint32_t)MLG_STATUS_CAPACITY);
    }
  }
}

// ------------------------------------------------------- one-launch build
//
// Small systems (n <= kFusedMaxAtoms, per-cell scans): the whole build in one
// cooperative launch, where the chain of small kernels above would be bound
// by launch latency.  CTA 0 alone bins the atoms (init, bounding box, cell
// histogram, cell scan, scatter) and then releases a flag; every CTA counts
// its (cell, split) items; a grid barrier; every CTA scans the kept counts
// into shared memory for its row starts (CTA 0 also writes row_ptr, n_edges
// and the capacity check) and fills its items, reusing the staged candidates
// of a cell it has just counted.  Both waits are bounded: a CTA whose wait
// runs out sets MLG_STATUS_TIMEOUT and leaves, which ends the others' waits
// the same way.  The launch is cooperative, so every CTA is resident.
constexpr int kFusedMaxAtoms = 4096;
constexpr long long kFusedSpinLimit = 1ll << 21;  // polls, 256 ns apart: a second or two

struct FusedSync {
  unsigned int ready;    // 1 once CTA 0 has binned the atoms
  unsigned int arrived;  // CTAs done with the count pass
};                       // zeroed by the host before each launch

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// polls until *p >= want; false if `polls` polls (0: kFusedSpinLimit) ran out first
__device__ __forceinline__ bool wait_at_least(const unsigned* p, unsigned want, long long polls) {
  const long long limit = polls > 0 ? polls : kFusedSpinLimit;
  for (long long it = 0; it < limit; ++it) {
    if (ld_acquire_gpu(p) >= want) return true;
    __nanosleep(256);
  }
  return false;
}

// Dynamic shared memory of the one-launch build: the per-cell scan's, then
// the row starts; CTA 0's binning scratch (histogram and three per-atom
// arrays) must fit in the same bytes.
template <int CAP>
__host__ __device__ constexpr size_t fused_build_smem(int64_t n) {
  return CellSmem<CAP>::bytes(true, true) + (size_t)(n + 1) * sizeof(int);
}
template <int CAP>
__host__ __device__ constexpr bool fused_build_fits(int64_t n, int ncell_cap) {
  return (size_t)(ncell_cap + 1 + 3 * n) * sizeof(int) <= fused_build_smem<CAP>(n);
}

template <int CAP>
__global__ void __launch_bounds__(kCellWarps * 32, 2)
    k_build_fused(BuildArgs a, BuildPlan p, int ncell_cap, int nsplit, FusedSync* sync) {
  if (gated_off(a.gate)) return;  // before any wait: every CTA leaves alike
  __shared__ CellGrid sg;
  __shared__ WarpScratch sws[kCellWarps];
  __shared__ int s_ok;
  extern __shared__ __align__(16) unsigned char s_dyn[];
  int* s_off = reinterpret_cast<int*>(s_dyn + CellSmem<CAP>::bytes(true, true));  // [n + 1] row starts
  const int tid = threadIdx.x;
  const unsigned tout = MLG_STATUS_TIMEOUT;

  if (blockIdx.x == 0) {
    // ---- binning, by this CTA alone, with its shared memory as scratch:
    // cell histogram (then starts), and each atom's cell, rank and image
    int* s_hist = reinterpret_cast<int*>(s_dyn);  // [ncell_cap + 1]
    int* s_cell = s_hist + ncell_cap + 1;          // [n]
    int* s_rank = s_cell + a.n;                    // [n]
    int* s_w = s_rank + a.n;                       // [n]
    for (int m = tid; m <= ncell_cap; m += blockDim.x) s_hist[m] = 0;
    if (tid < 3) {
      a.bbox[tid] = ~0ull;
      a.bbox[3 + tid] = 0ull;
    }
    if (tid == 0) {
      *a.n_truncated = 0;
      *a.status = 0u;
    }
    __syncthreads();
    if (p.any_open) {
      bbox_accumulate(a, p, tid, blockDim.x);
      __syncthreads();
    }
    if (tid == 0) {
      sg = derive_grid(p, a.bbox);
      *a.grid = sg;
    }
    __syncthreads();
    for (int64_t base = 0; base < a.n; base += blockDim.x)
      bin_atom(a, sg, base + tid, s_hist, s_rank, s_cell, s_w);
    __syncthreads();
    // cell starts: exclusive scan of the histogram, contiguous chunks per thread
    {
      const int per = (ncell_cap + (int)blockDim.x - 1) / (int)blockDim.x;
      const int m0 = tid * per, m1 = min(m0 + per, ncell_cap);
      int sum = 0;
      for (int m = m0; m < m1; ++m) sum += s_hist[m];
      int total;
      int off = block_excl_scan<int>(sum, &total);
      for (int m = m0; m < m1; ++m) {
        const int c = s_hist[m];
        s_hist[m] = off;
        a.cell_start[m] = off;
        off += c;
      }
      if (tid == 0) {
        s_hist[ncell_cap] = total;
        a.cell_start[ncell_cap] = total;
      }
    }
    __syncthreads();
    for (int64_t i = tid; i < a.n; i += blockDim.x) {
      const int cell = s_cell[i];
      if (cell >= 0) scatter_atom_at(a, sg, i, s_hist[cell] + s_rank[i], s_w[i]);
    }
    __syncthreads();
    if (tid == 0 && !a.hold_release) {
      __threadfence();
      st_release_gpu(&sync->ready, 1u);
    }
  }
  if (tid == 0) {
    s_ok = blockIdx.x == 0 ? 1 : (wait_at_least(&sync->ready, 1u, a.spin_polls) ? 1 : 0);
    if (s_ok && blockIdx.x != 0) sg = *a.grid;
    reinterpret_cast<CellStageT<CAP>*>(s_dyn)->staged_cell = -1;
  }
  __syncthreads();
  if (!s_ok) {
    if (tid == 0) atomicOr(a.status, tout);
    return;
  }

  // ---- count pass (keys kept for the fill)
  const int nitems = sg.ncell * nsplit;
  for (int item = blockIdx.x; item < nitems; item += gridDim.x)
    cellscan_item<false, true, true, CAP>(a, sg, sws, s_dyn, item / nsplit, item % nsplit,
                                          nsplit, nullptr);

  // ---- grid barrier: every count is written
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    atomicAdd(&sync->arrived, 1u);
    s_ok = wait_at_least(&sync->arrived, gridDim.x, a.spin_polls) ? 1 : 0;
  }
  __syncthreads();
  if (!s_ok) {
    if (tid == 0) atomicOr(a.status, tout);
    return;
  }

  // ---- row starts of every centre, then the fill pass
  scan_block<int>(a.kept, a.n, s_off, ScanTail{nullptr, nullptr, 0});
  if (blockIdx.x == 0)
    scan_block<long long>(a.kept, a.n, reinterpret_cast<long long*>(a.row_ptr),
                          ScanTail{a.n_edges, a.status, a.capacity});
  __syncthreads();
  for (int item = blockIdx.x; item < nitems; item += gridDim.x)
    cellscan_item<true, true, true, CAP>(a, sg, sws, s_dyn, item / nsplit, item % nsplit,
                                         nsplit, s_off);
}

}  // namespace mlg
