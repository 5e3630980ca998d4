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

// 32 channels (one lane per channel): one warp per centre, no block-wide
// barriers.  The weights stay in shared memory for the launch (Wk rows padded
// to 33 so that a warp reading a column touches 32 banks).  Per centre:
//   q = x Wq and u^h from shuffles of x and q;
//   logits four edges at a time: each lane holds g_b[lane] u^h[lane] for the
//   4 H (edge, head) pairs, and one butterfly reduce-scatter (M - 1
//   shuffles for M values, instead of 5 per value) leaves pair (l >> 1) of
//   the M = 4 H in lanes l and l ^ 1 (for H = 4);
//   softmax per head over the edges; z^h[lane] = sum_b P_b^h g_b[lane] (the
//   edge rows read again, now from L1); out[lane] = z^{h(lane)} . Wv[:, lane].
template <int M, typename T>
__device__ __forceinline__ T reduce_scatter(T (&v)[M], int lane) {
  // after the step with offset o = 16 / 2^s the lane keeps half of its values
  // (the upper half when lane & o is set) with its partner's matching half added
#pragma unroll
  for (int s = 0, cnt = M; cnt > 1; ++s, cnt >>= 1) {
    const int o = 16 >> s;
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < cnt / 2; ++j) {
      const T send = up ? v[j] : v[j + cnt / 2];
      const T keep = up ? v[j + cnt / 2] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  T r = v[0];
  // the lanes that still share a value (offsets below 32 / M) add up
#pragma unroll
  for (int o = 16 / M; o >= 1; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
  return r;
}

constexpr int kLocalW32Warps = 8;

template <typename T, int H>
inline size_t local_w32_smem(int nnei_max) {
  return ((size_t)32 * 32 * 2 + (size_t)32 * 33 +
          (size_t)kLocalW32Warps * ((size_t)H * nnei_max + (size_t)H * 33)) * sizeof(T);
}

template <typename T, int H>
__global__ void __launch_bounds__(kLocalW32Warps * 32) k_local_attn_w32(LocalArgs a) {
  constexpr int C = 32, D = C / H, M = 4 * H;
  extern __shared__ __align__(16) unsigned char smem_lw[];
  const int NM = a.nnei_max;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  T* sWq = reinterpret_cast<T*>(smem_lw);     // [32][32]
  T* sWv = sWq + C * C;                        // [32][32]
  T* sWk = sWv + C * C;                        // [32][33]
  T* sp = sWk + C * (C + 1) + (size_t)warp * (H * NM + H * (C + 1));  // [H][NM] logits, weights
  T* sz = sp + (size_t)H * NM;                 // [H][33] z^h
  const T* Hn = static_cast<const T*>(a.H);
  const T* G = static_cast<const T*>(a.G);
  T* out = static_cast<T*>(a.out);
  for (int e = tid; e < C * C; e += blockDim.x) {
    sWq[e] = static_cast<const T*>(a.Wq)[e];
    sWv[e] = static_cast<const T*>(a.Wv)[e];
    sWk[(e / C) * (C + 1) + e % C] = static_cast<const T*>(a.Wk)[e];
  }
  __syncthreads();
  const int64_t E = a.row_ptr[a.n_centres];
  if (E > a.capacity || (*a.status & MLG_STATUS_CAPACITY)) return;
  const T rsd = (T)(1.0 / sqrt((double)D));
  for (int64_t i = (int64_t)blockIdx.x * kLocalW32Warps + warp; i < a.n_centres;
       i += (int64_t)gridDim.x * kLocalW32Warps) {
    const int64_t b0 = a.row_ptr[i];
    const int n = (int)(a.row_ptr[i + 1] - b0);
    if (n <= 0 || n > NM) {  // no edges: a zero row; longer than nnei_max: flagged
      out[i * C + lane] = T(0);
      if (n > NM && lane == 0) atomicOr(a.status, (uint32_t)MLG_STATUS_ROW_TOO_LONG);
      continue;
    }
    const T x = Hn[i * C + lane];
    T q = T(0);
#pragma unroll
    for (int k = 0; k < C; ++k) q = fma(__shfl_sync(0xffffffffu, x, k), sWq[k * C + lane], q);
    T u[H];
#pragma unroll
    for (int h = 0; h < H; ++h) {
      u[h] = T(0);
#pragma unroll
      for (int t = 0; t < D; ++t)
        u[h] = fma(sWk[lane * (C + 1) + h * D + t], __shfl_sync(0xffffffffu, q, h * D + t), u[h]);
    }
    // logits, four edges at a time
    const int pidx = (lane / (32 / M)) % M;   // the (edge, head) pair this lane ends with
    for (int bb = 0; bb < n; bb += 4) {
      T v[M];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const T g = bb + e < n ? G[(b0 + bb + e) * C + lane] : T(0);
#pragma unroll
        for (int h = 0; h < H; ++h) v[e * H + h] = g * u[h];
      }
      const T r = reduce_scatter<M>(v, lane);
      const int e = pidx / H, h = pidx % H;
      if (lane % (32 / M) == 0 && bb + e < n)
        sp[h * NM + bb + e] = (T)a.sw[b0 + bb + e] * r * rsd;
    }
    __syncwarp();
    // softmax over the edges, per head
#pragma unroll
    for (int h = 0; h < H; ++h) {
      T* ph = sp + h * NM;
      T mx = -INFINITY;
      for (int b = lane; b < n; b += 32) mx = fmax(mx, ph[b]);
      for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      T l = T(0);
      for (int b = lane; b < n; b += 32) {
        const T ev = exp_t<T>(ph[b] - mx);
        ph[b] = ev;
        l += ev;
      }
      l = warp_sum(l);
      const T inv = T(1) / l;
      for (int b = lane; b < n; b += 32) ph[b] *= inv;
    }
    __syncwarp();
    // z^h[lane] = sum_b P_b^h g_b[lane]
    T z[H];
#pragma unroll
    for (int h = 0; h < H; ++h) z[h] = T(0);
    for (int b = 0; b < n; ++b) {
      const T g = G[(b0 + b) * C + lane];
#pragma unroll
      for (int h = 0; h < H; ++h) z[h] = fma(sp[h * NM + b], g, z[h]);
    }
#pragma unroll
    for (int h = 0; h < H; ++h) sz[h * (C + 1) + lane] = z[h];
    __syncwarp();
    // out[lane] = z^{h(lane)} . Wv[:, lane]
    const T* zh = sz + (lane / D) * (C + 1);
    T o = T(0);
#pragma unroll
    for (int k = 0; k < C; ++k) o = fma(zh[k], sWv[k * C + lane], o);
    out[i * C + lane] = o;
    __syncwarp();  // the next centre reuses sp and sz
  }
}

}  // namespace mlg
