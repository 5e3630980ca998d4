// mlg_verlet.cuh -- Verlet-skin reuse of the neighbour search across MD
// steps (sm_100a).
//
// The deepmd-kit issue "DPA4 .pt2 LAMMPS (C++ AOTI) inference 3-6x slower
// than Python (ASE)" proposes (Proposed optimizations) to keep the device
// tensors of the edge construction while the neighbour list is unchanged,
// and to rebuild when the MD engine's skin criterion asks for it.  Here:
//
//   candidate list  the destination CSR at rcut + skin, built by the regular
//                   build (cap kVerletListCap, canonical order), together
//                   with the coordinates it was built at;
//   check           a device reduction of the largest displacement since
//                   then: once some atom has moved skin / 2 or more (or a
//                   coordinate is not finite, or no list exists yet) a
//                   device word asks for a rebuild, and the build kernels,
//                   gated on that word, run; otherwise they return at once.
//                   No host round trip decides anything.
//   refine          every candidate (source, shift) re-evaluated at the
//                   current coordinates with the build's own operation
//                   order, kept if r < rcut, capped to the nnei_max nearest
//                   by (r^2, source, shift) and written in canonical order.
//
// While no atom has moved skin / 2, every pair within rcut at the current
// positions was within rcut + skin at the list's positions (triangle
// inequality), and the candidates are already in canonical (source, shift)
// order, so the refined CSR is the full build's, bit for bit.  The cap
// cannot be applied to the list itself: the nearest nnei_max at the old
// positions need not be the nearest now.
#pragma once

#include "mlg_common.cuh"
#include "mlg_build.cuh"

namespace mlg {

constexpr int kVerletListCap = 256;  // candidates kept per destination in the list
constexpr int kRefineWarps = 8;

struct VerletCheckArgs {
  int64_t n;
  const double* coords;       // current [n][3]
  const double* coords_ref;   // the list's [n][3]
  const uint32_t* state;      // list state word (bit 0: the list is valid)
  double skin;
  uint32_t* gate;             // out: 1 = rebuild the list in this step
  unsigned long long* dmax;   // scratch, zero on entry: bits of the largest squared move
  unsigned int* done;         // scratch, zero on entry: CTAs finished
  uint32_t* out_status;       // the refined CSR's status and truncation count, reset here
  int64_t* out_trunc;
};

// Largest squared displacement on the raw coordinates (an atom re-wrapped
// into the box has moved by a box length); a non-finite one counts as
// infinite.  The last CTA to finish takes the decision (no CTA waits).
__global__ void __launch_bounds__(256) k_verlet_check(VerletCheckArgs a) {
  __shared__ double s_max[8];
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *a.out_status = 0u;
    *a.out_trunc = 0;
  }
  double m = 0.0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < a.n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const double dx = __dsub_rn(a.coords[3 * i], a.coords_ref[3 * i]);
    const double dy = __dsub_rn(a.coords[3 * i + 1], a.coords_ref[3 * i + 1]);
    const double dz = __dsub_rn(a.coords[3 * i + 2], a.coords_ref[3 * i + 2]);
    double d2 = __dadd_rn(__dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy)), __dmul_rn(dz, dz));
    if (!(d2 <= 1.79e308)) d2 = INFINITY;  // NaN or overflow
    m = fmax(m, d2);
  }
  m = warp_max(m);
  if (lane_id() == 0) s_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmax(m, s_max[w]);
    // non-negative doubles order like their bit patterns
    atomicMax(a.dmax, (unsigned long long)__double_as_longlong(m));
    __threadfence();
    const unsigned prev = atomicAdd(a.done, 1u);
    if (prev == gridDim.x - 1) {
      __threadfence();
      const double mx = __longlong_as_double((long long)atomicAdd(a.dmax, 0ull));
      const bool valid = (*a.state & 1u) != 0u;
      const bool moved = !(__dmul_rn(2.0, __dsqrt_rn(mx)) < a.skin);
      *a.gate = (!valid || moved) ? 1u : 0u;
    }
  }
}

// After a gated rebuild: the list's coordinates and state.
__global__ void k_verlet_commit(const uint32_t* gate, int64_t n, const double* coords,
                                double* coords_ref, uint32_t* state, int64_t* n_builds) {
  if (*gate == 0u) return;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < 3 * n;
       t += (int64_t)gridDim.x * blockDim.x)
    coords_ref[t] = coords[t];
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *state |= 1u;
    *n_builds += 1;
  }
}

struct RefineArgs {
  int64_t n;
  const double* coords;
  double box[9];
  double rcut, r_on, rc2;
  int nnei_max;
  double taylor[12];
  // candidate list
  const int64_t* cp;
  const int32_t* cs;
  const int32_t* ch;
  const uint32_t* cand_status;
  const int64_t* cand_trunc;
  // per-destination counts (workspace)
  int* kept;
  int* raw;
  // the refined CSR
  int64_t capacity;
  int64_t* row_ptr;
  int32_t* src;
  int32_t* shift;
  double* vec;
  double* dist;
  double* sw;
  int64_t* n_truncated;
  uint32_t* status;
};

// r^2 of candidate c of destination i (coordinates xi) at the current
// positions, with the vector in v (the build's edge_vec order).
__device__ __forceinline__ double refine_r2(const RefineArgs& a, const double* xi, int64_t c,
                                            int* j, int* S, double* v) {
  *j = a.cs[c];
  S[0] = a.ch[3 * c];
  S[1] = a.ch[3 * c + 1];
  S[2] = a.ch[3 * c + 2];
  const double xj[3] = {a.coords[3 * (int64_t)*j], a.coords[3 * (int64_t)*j + 1],
                        a.coords[3 * (int64_t)*j + 2]};
  return edge_vec(a.box, xi, xj, S, v);
}

__device__ __forceinline__ void refine_write(const RefineArgs& a, int64_t p, int j, const int* S,
                                             const double* v, double r2) {
  if (p >= a.capacity) return;
  const double r = __dsqrt_rn(r2);
  a.src[p] = j;
  a.shift[3 * p] = S[0];
  a.shift[3 * p + 1] = S[1];
  a.shift[3 * p + 2] = S[2];
  a.vec[3 * p] = v[0];
  a.vec[3 * p + 1] = v[1];
  a.vec[3 * p + 2] = v[2];
  a.dist[p] = r;
  a.sw[p] = switch_fn(r, a.rcut, a.r_on, a.taylor);
}

// Warp per destination: how many candidates lie within rcut now.
__global__ void __launch_bounds__(kRefineWarps * 32) k_refine_count(RefineArgs a) {
  __shared__ int s_trunc;
  if (threadIdx.x == 0) s_trunc = 0;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    // what the list's build found about the input, and whether the list is whole
    const uint32_t cst = *a.cand_status;
    uint32_t st = cst & (MLG_STATUS_NONFINITE_COORD | MLG_STATUS_TYPE_RANGE |
                         MLG_STATUS_IMAGE_RANGE | MLG_STATUS_INTERNAL | MLG_STATUS_TIMEOUT);
    if ((cst & MLG_STATUS_CAPACITY) || *a.cand_trunc != 0) st |= MLG_STATUS_LIST_INCOMPLETE;
    if (st) atomicOr(a.status, st);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int64_t i = (int64_t)blockIdx.x * kRefineWarps + warp;
  if (i < a.n) {
    const double xi[3] = {a.coords[3 * i], a.coords[3 * i + 1], a.coords[3 * i + 2]};
    const int64_t c0 = a.cp[i], c1 = a.cp[i + 1];
    int cnt = 0;
    for (int64_t c = c0 + lane; c < c1; c += 32) {
      int j, S[3];
      double v[3];
      cnt += refine_r2(a, xi, c, &j, S, v) < a.rc2 ? 1 : 0;
    }
    cnt = warp_sum(cnt);
    if (lane == 0) {
      a.raw[i] = cnt;
      a.kept[i] = cnt < a.nnei_max ? cnt : a.nnei_max;
      if (cnt > a.nnei_max) atomicAdd(&s_trunc, 1);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_trunc)
    atomicAdd((unsigned long long*)a.n_truncated, (unsigned long long)s_trunc);
}

// Warp per destination: write the kept candidates.  Rows within the cap keep
// every accepted candidate in list order (already canonical); longer rows
// keep the nnei_max smallest (r^2 bits, candidate index), which is the
// build's (r^2, source, shift) order, and write them in index order.
__global__ void __launch_bounds__(kRefineWarps * 32) k_refine_fill(RefineArgs a) {
  __shared__ unsigned long long s_keys[kRefineWarps][2][kVerletListCap];
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int64_t i = (int64_t)blockIdx.x * kRefineWarps + warp;
  if (i >= a.n) return;
  const int n = a.kept[i];
  if (n == 0) return;
  const int raw = a.raw[i];
  const int64_t p0 = a.row_ptr[i];
  const double xi[3] = {a.coords[3 * i], a.coords[3 * i + 1], a.coords[3 * i + 2]};
  const int64_t c0 = a.cp[i], c1 = a.cp[i + 1];
  if (raw <= a.nnei_max) {
    int pos = 0;
    for (int64_t base = c0; base < c1; base += 32) {
      const int64_t c = base + lane;
      int j = 0, S[3] = {0, 0, 0};
      double v[3] = {0.0, 0.0, 0.0}, r2 = 0.0;
      bool acc = false;
      if (c < c1) {
        r2 = refine_r2(a, xi, c, &j, S, v);
        acc = r2 < a.rc2;
      }
      const unsigned m = __ballot_sync(kFull, acc);
      if (acc) refine_write(a, p0 + pos + __popc(m & lanemask_lt()), j, S, v, r2);
      pos += __popc(m);
    }
    return;
  }
  // truncated row: at most kVerletListCap candidates (the list's own cap)
  unsigned long long* keys = s_keys[warp][0];
  unsigned long long* d2 = s_keys[warp][1];
  int pos = 0;
  for (int64_t base = c0; base < c1; base += 32) {
    const int64_t c = base + lane;
    bool acc = false;
    double r2 = 0.0;
    if (c < c1) {
      int j, S[3];
      double v[3];
      r2 = refine_r2(a, xi, c, &j, S, v);
      acc = r2 < a.rc2;
    }
    const unsigned m = __ballot_sync(kFull, acc);
    if (acc) {
      const int q = pos + __popc(m & lanemask_lt());
      if (q < kVerletListCap) {
        keys[q] = (unsigned long long)(c - c0);
        d2[q] = (unsigned long long)__double_as_longlong(r2);
      }
    }
    pos += __popc(m);
  }
  __syncwarp();
  const int cnt = pos < kVerletListCap ? pos : kVerletListCap;
  const int keep = n < cnt ? n : cnt;
  if (keep != n && lane == 0) atomicOr(a.status, (uint32_t)MLG_STATUS_INTERNAL);
  warp_sort_pairs(d2, keys, cnt);
  warp_sort_keys(keys, keep);
  for (int e = lane; e < keep; e += 32) {
    int j, S[3];
    double v[3];
    const double r2 = refine_r2(a, xi, c0 + (int64_t)keys[e], &j, S, v);
    refine_write(a, p0 + e, j, S, v, r2);
  }
}

}  // namespace mlg
