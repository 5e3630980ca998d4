// mlg_attn.cuh -- stage 2: block-dense per-centre multi-head attention over
// the destination CSR (sm_100a).
//
// deepmd-kit issue "NeighborGraph attention is 4-9x slower than dense and
// OOM-prone", Proposed fix: each centre's edge features are collected into
// one small block by way of destination_row_ptr, attended to with the same
// batched products the dense route uses per centre (Root cause), the unequal
// row lengths handled by masking each row, and the outputs returned to their
// edges.  Here the gather is the contiguous CSR slab of the centre, the
// "mask" is the loop bound n_i, and the scatter is a contiguous slab store:
// no (sum nnei^2, c) tensor and no Q/K/V tensor ever reaches global memory.
//
// Per centre i (edges a, b < n), per head h (columns h d .. h d + d):
//   q_a = G_a Wq, k_b = G_b Wk, v_b = G_b Wv
//   l_ab = s_a s_b (q_a . k_b) / sqrt(d)
//   O_a = sum_b exp(l_ab - m_a) v_b / sum_b exp(l_ab - m_a),  m_a = max_b l_ab
// With `smooth` (slot-occupancy softmax, NeighborGraph issue, Numerics note:
// the denominator counts empty slots as phantoms), the centre's
// phi = nnei_max - n padded slots take part as phantoms of logit 0 and value
// 0: m_a = max(max_b l_ab, 0) and the denominator gains phi exp(-m_a).
#pragma once

#include "mlg_common.cuh"

namespace mlg {

struct AttnArgs {
  const int64_t* row_ptr;
  const double* sw;
  int64_t n_centres;
  int64_t capacity;
  int nnei_max;
  int C, H, D;
  const void* G;
  void* out;
  const void* Wq;
  const void* Wk;
  const void* Wv;
  uint32_t* status;
  int min_n;  // only centres with more than min_n edges (0: all)
  int smooth;  // slot-occupancy softmax (phantom slots up to nnei_max)
};

template <typename T>
__device__ __forceinline__ T fast_exp(T x);
template <>
__device__ __forceinline__ float fast_exp<float>(float x) { return __expf(x); }
template <>
__device__ __forceinline__ double fast_exp<double>(double x) { return exp(x); }

constexpr int kAttnWarps = 8;

// Generic kernel: one CTA per centre (grid-stride), one head at a time.
// Shared memory: Q, K, V of the head [nnei_max][d + 1] each, s [nnei_max],
// one probability row per warp [kAttnWarps][nnei_max].
template <typename T>
__global__ void __launch_bounds__(kAttnWarps * 32) k_attn_generic(AttnArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* sm = reinterpret_cast<T*>(smem_raw);
  const int C = a.C, D = a.D, DP = a.D + 1, NM = a.nnei_max;
  T* sQ = sm;
  T* sK = sQ + (size_t)NM * DP;
  T* sV = sK + (size_t)NM * DP;
  T* sS = sV + (size_t)NM * DP;
  T* sP = sS + NM;
  const T* G = static_cast<const T*>(a.G);
  T* out = static_cast<T*>(a.out);
  const T* W3[3] = {static_cast<const T*>(a.Wq), static_cast<const T*>(a.Wk),
                    static_cast<const T*>(a.Wv)};
  if (*a.status & MLG_STATUS_CAPACITY) return;
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const T rsd = T(1) / sqrt(T(D));
  for (int64_t i = blockIdx.x; i < a.n_centres; i += gridDim.x) {
    const int64_t base = a.row_ptr[i];
    const int n = (int)(a.row_ptr[i + 1] - base);
    if (n > NM) {  // longer than the caller's nnei_max: not written, flagged
      if (threadIdx.x == 0) atomicOr(a.status, (uint32_t)MLG_STATUS_ROW_TOO_LONG);
      continue;
    }
    if (n <= a.min_n || base + n > a.capacity) continue;
    for (int t = threadIdx.x; t < n; t += blockDim.x) sS[t] = (T)a.sw[base + t];
    __syncthreads();
    for (int h = 0; h < a.H; ++h) {
      // projections of this head: 3 d outputs per edge row
      for (int o = threadIdx.x; o < n * 3 * D; o += blockDim.x) {
        const int row = o / (3 * D), m = o - row * 3 * D;
        const int which = m / D, t = m - which * D;
        const T* W = W3[which];
        const T* g = G + (base + row) * C;
        const int col = h * D + t;
        T acc = T(0);
        for (int k = 0; k < C; ++k) acc += g[k] * W[(size_t)k * C + col];
        T* dst = which == 0 ? sQ : (which == 1 ? sK : sV);
        if (which == 0) acc *= sS[row] * rsd;
        if (which == 1) acc *= sS[row];
        dst[row * DP + t] = acc;
      }
      __syncthreads();
      // one warp per query row: logits, softmax, AV
      T* p = sP + (size_t)warp * NM;
      const int phi = a.smooth ? NM - n : 0;  // phantom slots of logit 0, value 0
      for (int r = warp; r < n; r += kAttnWarps) {
        T mx = phi > 0 ? T(0) : -INFINITY;
        for (int b = lane; b < n; b += 32) {
          T l = T(0);
          for (int t = 0; t < D; ++t) l += sQ[r * DP + t] * sK[b * DP + t];
          p[b] = l;
          mx = l > mx ? l : mx;
        }
        mx = warp_max(mx);
        T z = T(0);
        for (int b = lane; b < n; b += 32) {
          T e = fast_exp<T>(p[b] - mx);
          p[b] = e;
          z += e;
        }
        z = warp_sum(z);
        if (phi > 0) z += T(phi) * fast_exp<T>(-mx);  // mx >= 0 here
        __syncwarp();
        const T rz = T(1) / z;
        for (int t = lane; t < D; t += 32) {
          T acc = T(0);
          for (int b = 0; b < n; ++b) acc += p[b] * sV[b * DP + t];
          out[(base + r) * C + h * D + t] = acc * rz;
        }
        __syncwarp();
      }
      __syncthreads();
    }
  }
}

template <typename T>
inline size_t attn_generic_smem(int nnei_max, int D) {
  return sizeof(T) * ((size_t)3 * nnei_max * (D + 1) + nnei_max + (size_t)kAttnWarps * nnei_max);
}

}  // namespace mlg
