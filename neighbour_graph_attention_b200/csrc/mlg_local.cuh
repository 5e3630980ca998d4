// mlg_local.cuh -- local attention, one query per centre (sm_100a).
//
// LocalAtten of the NeighborGraph issue ("Graph-native alternatives", item 2:
// per-centre CSR segments with queries = centres and keys = edges): for
// centre i, q = H_i Wq from its own feature row, keys and values from its
// edges, per head l_b = s_b (q . k_b) / sqrt(d), softmax over the centre's
// edges, out_i = sum_b P_b v_b, heads concatenated; a centre without edges
// gets a zero row.
//
// With a single query the products reassociate so that K and V are never
// formed:
//   l_b^h  = s_b (G_b . u^h) / sqrt(d),   u^h = Wk[:, head h] q^h   (c x d per head)
//   out^h  = z^h Wv[:, head h],            z^h = sum_b P_b^h G_b    (c per head)
// 3 c^2 + 2 n c H multiply-adds per centre instead of about 2 n c^2.  One CTA
// works on one centre at a time (grid-stride over centres); the centre's
// row, q, u, the weights P and z live in shared memory; G rows are read from
// global memory (each twice, the second time mostly from L1).
#pragma once

#include "mlg_common.cuh"

namespace mlg {

struct LocalArgs {
  const int64_t* row_ptr;
  const double* sw;
  int64_t n_centres;
  int64_t capacity;
  int channels;
  int heads;
  int nnei_max;
  const void* H;   // [n_centres][c]
  const void* G;   // [E][c]
  void* out;       // [n_centres][c]
  const void* Wq;  // [c][c], y = x W
  const void* Wk;
  const void* Wv;
  uint32_t* status;
};

constexpr int kLocalThreads = 256;
constexpr int kLocalMaxC = 256;  // channels: at most 8 per lane in the logit pass

template <typename T>
inline size_t local_smem(int c, int heads, int nnei_max) {
  return ((size_t)2 * c + (size_t)2 * heads * c + (size_t)heads * nnei_max) * sizeof(T);
}

template <typename T>
__device__ __forceinline__ T exp_t(T x);
template <>
__device__ __forceinline__ double exp_t<double>(double x) { return exp(x); }
template <>
__device__ __forceinline__ float exp_t<float>(float x) { return expf(x); }

template <typename T>
__global__ void __launch_bounds__(kLocalThreads) k_local_attn(LocalArgs a) {
  extern __shared__ __align__(16) unsigned char smem_local[];
  const int c = a.channels, H = a.heads, d = c / H, NM = a.nnei_max;
  T* sx = reinterpret_cast<T*>(smem_local);  // [c]     the centre's feature row
  T* sq = sx + c;                             // [c]     q = x Wq
  T* su = sq + c;                             // [H][c]  u^h
  T* sz = su + (size_t)H * c;                 // [H][c]  z^h
  T* sp = sz + (size_t)H * c;                 // [H][NM] logits, then weights
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, NW = blockDim.x >> 5;
  const T* Hn = static_cast<const T*>(a.H);
  const T* G = static_cast<const T*>(a.G);
  T* out = static_cast<T*>(a.out);
  const T* Wq = static_cast<const T*>(a.Wq);
  const T* Wk = static_cast<const T*>(a.Wk);
  const T* Wv = static_cast<const T*>(a.Wv);
  const int64_t E = a.row_ptr[a.n_centres];
  if (E > a.capacity || (*a.status & MLG_STATUS_CAPACITY)) return;
  const T rsd = (T)(1.0 / sqrt((double)d));

  for (int64_t i = blockIdx.x; i < a.n_centres; i += gridDim.x) {
    const int64_t b0 = a.row_ptr[i];
    const int n = (int)(a.row_ptr[i + 1] - b0);
    T* orow = out + i * c;
    if (n <= 0 || n > NM) {  // no edges: a zero row; longer than nnei_max: flagged
      for (int m = tid; m < c; m += blockDim.x) orow[m] = T(0);
      if (n > NM && tid == 0) atomicOr(a.status, (uint32_t)MLG_STATUS_ROW_TOO_LONG);
      continue;
    }
    for (int m = tid; m < c; m += blockDim.x) sx[m] = Hn[i * c + m];
    __syncthreads();
    // q = x Wq
    for (int m = tid; m < c; m += blockDim.x) {
      T acc = T(0);
      for (int k = 0; k < c; ++k) acc = fma(sx[k], Wq[(size_t)k * c + m], acc);
      sq[m] = acc;
    }
    __syncthreads();
    // u^h[k] = sum_t Wk[k][h d + t] q[h d + t]
    for (int e = tid; e < H * c; e += blockDim.x) {
      const int h = e / c, k = e - h * c;
      const T* wr = Wk + (size_t)k * c + h * d;
      T acc = T(0);
      for (int t = 0; t < d; ++t) acc = fma(wr[t], sq[h * d + t], acc);
      su[e] = acc;
    }
    __syncthreads();
    // logits: one warp per edge, the edge's row in registers
    for (int b = warp; b < n; b += NW) {
      const T* gb = G + (b0 + b) * c;
      T g[kLocalMaxC / 32];
#pragma unroll
      for (int r = 0; r < kLocalMaxC / 32; ++r) g[r] = lane + 32 * r < c ? gb[lane + 32 * r] : T(0);
      const T sb = (T)a.sw[b0 + b];
      for (int h = 0; h < H; ++h) {
        T acc = T(0);
#pragma unroll
        for (int r = 0; r < kLocalMaxC / 32; ++r)
          if (lane + 32 * r < c) acc = fma(g[r], su[h * c + lane + 32 * r], acc);
        acc = warp_sum(acc);
        if (lane == 0) sp[h * NM + b] = sb * acc * rsd;
      }
    }
    __syncthreads();
    // softmax over the edges, one warp per head
    for (int h = warp; h < H; h += NW) {
      T* ph = sp + h * NM;
      T mx = -INFINITY;
      for (int b = lane; b < n; b += 32) mx = fmax(mx, ph[b]);
      for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(kFull, mx, o));
      T l = T(0);
      for (int b = lane; b < n; b += 32) {
        const T e = exp_t<T>(ph[b] - mx);
        ph[b] = e;
        l += e;
      }
      l = warp_sum(l);
      const T inv = T(1) / l;
      for (int b = lane; b < n; b += 32) ph[b] *= inv;
    }
    __syncthreads();
    // z^h[k] = sum_b P_b^h G_b[k]
    for (int e = tid; e < H * c; e += blockDim.x) {
      const int h = e / c, k = e - h * c;
      const T* ph = sp + h * NM;
      T acc = T(0);
      for (int b = 0; b < n; ++b) acc = fma(ph[b], G[(b0 + b) * c + k], acc);
      sz[e] = acc;
    }
    __syncthreads();
    // out[m] = sum_k z^h[k] Wv[k][m], h = head of column m
    for (int m = tid; m < c; m += blockDim.x) {
      const T* zh = sz + (m / d) * c;
      T acc = T(0);
      for (int k = 0; k < c; ++k) acc = fma(zh[k], Wv[(size_t)k * c + m], acc);
      orow[m] = acc;
    }
    __syncthreads();  // the next centre reuses the shared arrays
  }
}

}  // namespace mlg
