// mlg_attn_hg.cuh -- block-dense attention for wide edge features (C = 128),
// one head group per CTA (sm_100a).
//
// Same per-centre attention as mlg_attn_tile.cuh (NeighborGraph issue,
// Proposed fix: dense attention math per centre, masks for the ragged tail,
// results back on the edge axis), for channel counts whose projection
// weights do not fit in shared memory.  The work splits over a 2-D grid:
// blockIdx.y picks a group of HG heads, so only that group's columns of
// [Wq | Wk | Wv] are needed; blockIdx.x is a persistent CTA that packs
// consecutive centres (one contiguous CSR slab) into tiles of at most R rows.
// Per tile:
//   1. QKV_g = X [rows][C] . W_g [C][3 HG d]: register-tiled GEMM whose
//      operands stream through shared memory in K chunks (cp.async, double
//      buffered; X and W stay L2-resident across head groups);
//   2. attention of the group's heads, one lane per (row, head), lanes of a
//      warp in lock-step over keys (broadcast reads), running-max softmax;
//   3. the group's output columns are written to global memory.
// One launch per layer (the layer's output must be complete before the next).
#pragma once

#include "mlg_common.cuh"
#include "mlg_attn_tile.cuh"

namespace mlg {

struct HgArgs {
  const int64_t* row_ptr;
  const double* sw;
  int64_t n_centres;
  int64_t capacity;
  int nnei_max;  // centres with more edges are skipped and flagged
  int smooth;    // slot-occupancy softmax (phantom slots up to nnei_max)
  const void* G;
  void* out;
  const void* Wq;
  const void* Wk;
  const void* Wv;
  uint32_t* status;
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <typename T, int C, int D, int HG, int R, int NT, int TM, int TN, int KC>
struct HgCfg {
  static constexpr int H = C / D;
  static constexpr int NG = H / HG;            // head groups
  static constexpr int GW = HG * D;            // columns of one of q/k/v in the group
  static constexpr int N3 = 3 * GW;            // GEMM output columns
  static constexpr int NCG = N3 / TN;
  static constexpr int NRG = R / TM;
  static constexpr int XS = KC + 16 / (int)sizeof(T);   // X chunk row stride (elements)
  static constexpr int QS = N3 + (sizeof(T) == 8 ? 1 : 4);
  static constexpr int MAXC = 64;
  static_assert(NCG * NRG == NT, "thread grid must cover the tile");
  static_assert(H % HG == 0 && C % KC == 0 && KC % 4 == 0, "shapes");
  static_assert(GW % NCG == 0 || NCG % GW == 0, "column groups and q/k/v blocks");
  static constexpr size_t XC_BYTES = (size_t)R * XS * sizeof(T);
  static constexpr size_t WC_BYTES = (size_t)KC * N3 * sizeof(T);
  static constexpr size_t OFF_X = 0;                       // [2][R][XS]
  static constexpr size_t OFF_W = OFF_X + 2 * XC_BYTES;    // [2][KC][N3]
  static constexpr size_t OFF_Q = OFF_W + 2 * WC_BYTES;    // [R][QS]
  static constexpr size_t OFF_S = OFF_Q + (size_t)R * QS * sizeof(T);
  static constexpr size_t OFF_META = (OFF_S + (size_t)R * sizeof(T) + 15) / 16 * 16;
  static constexpr size_t SMEM = OFF_META + sizeof(TileMeta);
};

template <typename T, int C, int D, int HG, int R, int NT, int TM, int TN, int KC>
__global__ void __launch_bounds__(NT) k_attn_hg(HgArgs a) {
  using Cfg = HgCfg<T, C, D, HG, R, NT, TM, TN, KC>;
  constexpr int GW = Cfg::GW, N3 = Cfg::N3, NCG = Cfg::NCG, XS = Cfg::XS, QS = Cfg::QS;
  extern __shared__ __align__(128) unsigned char smem[];
  T* sXc = reinterpret_cast<T*>(smem + Cfg::OFF_X);
  T* sWc = reinterpret_cast<T*>(smem + Cfg::OFF_W);
  T* sQ = reinterpret_cast<T*>(smem + Cfg::OFF_Q);
  T* sS = reinterpret_cast<T*>(smem + Cfg::OFF_S);
  TileMeta& meta = *reinterpret_cast<TileMeta*>(smem + Cfg::OFF_META);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y;                    // head group
  const T* G = static_cast<const T*>(a.G);
  T* out = static_cast<T*>(a.out);
  const T* Wm[3] = {static_cast<const T*>(a.Wq), static_cast<const T*>(a.Wk),
                    static_cast<const T*>(a.Wv)};
  const int64_t E = a.row_ptr[a.n_centres];
  if (E > a.capacity || (*a.status & MLG_STATUS_CAPACITY)) return;

  if (tid == 0) {
    const int64_t r0 = E * blockIdx.x / gridDim.x, r1 = E * (blockIdx.x + 1) / gridDim.x;
    auto lb = [&](int64_t r) {
      int64_t lo = 0, hi = a.n_centres;
      while (lo < hi) {
        int64_t mid = (lo + hi) >> 1;
        if (a.row_ptr[mid] < r) lo = mid + 1; else hi = mid;
      }
      return (int)lo;
    };
    meta.next_c = lb(r0);
    meta.c_end = blockIdx.x + 1 == gridDim.x ? (int)a.n_centres : lb(r1);
  }
  __syncthreads();

  const T qscale = sizeof(T) == 4 ? T(1.4426950408889634 / sqrt((double)D))
                                  : T(1.0 / sqrt((double)D));
  while (true) {
    // ---- plan the next tile (thread 0), centres with more than R edges skipped
    if (tid == 0) {
      int c = meta.next_c, k = 0, rows = 0, tasks = 0;
      const int c_end = meta.c_end;
      while (c < c_end) {
        int n = (int)(a.row_ptr[c + 1] - a.row_ptr[c]);
        if (n > 0 && n <= R && n <= a.nnei_max) break;
        if (n > a.nnei_max && g == 0) atomicOr(a.status, (uint32_t)MLG_STATUS_ROW_TOO_LONG);
        ++c;
      }
      meta.row0[0] = c < c_end ? a.row_ptr[c] : 0;
      while (c < c_end && k < Cfg::MAXC) {
        int n = (int)(a.row_ptr[c + 1] - a.row_ptr[c]);
        if (n > R || n > a.nnei_max || rows + n > R) break;
        meta.off[0][k] = rows;
        meta.task0[0][k] = tasks;
        tasks += (n * HG + 31) / 32;
        rows += n;
        ++k;
        ++c;
      }
      meta.off[0][k] = rows;
      meta.task0[0][k] = tasks;
      meta.ncent[0] = k;
      meta.nrows[0] = rows;
      meta.next_c = c;
    }
    __syncthreads();
    const int rows = meta.nrows[0];
    const int64_t row0 = meta.row0[0];
    if (rows == 0) break;
    for (int t = tid; t < rows; t += NT) sS[t] = (T)a.sw[row0 + t];

    // ---- 1. GEMM over K chunks
    auto stage = [&](int kc, int b) {
      const int k0 = kc * KC;
      T* xd = sXc + (size_t)b * R * XS;
      constexpr int XV = KC * (int)sizeof(T) / 16;        // 16-byte pieces per row chunk
      for (int e = tid; e < rows * XV; e += NT) {
        const int r = e / XV, v = e - r * XV;
        cp_async16(xd + r * XS + v * (16 / (int)sizeof(T)),
                   G + (row0 + r) * C + k0 + v * (16 / (int)sizeof(T)));
      }
      T* wd = sWc + (size_t)b * KC * N3;
      constexpr int WV = GW * (int)sizeof(T) / 16;        // pieces per row of one matrix
      for (int e = tid; e < 3 * KC * WV; e += NT) {
        const int m = e / (KC * WV), rem = e - m * KC * WV;
        const int k = rem / WV, v = rem - k * WV;
        cp_async16(wd + k * N3 + m * GW + v * (16 / (int)sizeof(T)),
                   Wm[m] + (size_t)(k0 + k) * C + g * GW + v * (16 / (int)sizeof(T)));
      }
      cp_async_commit();
    };
    const int rg = tid / NCG, cg = tid % NCG;
    T acc[TM][TN];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) acc[i][j] = T(0);
    stage(0, 0);
    constexpr int NK = C / KC;
    for (int kc = 0; kc < NK; ++kc) {
      if (kc + 1 < NK) {
        stage(kc + 1, (kc + 1) & 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const T* xr = sXc + (size_t)(kc & 1) * R * XS + (rg * TM) * XS;
      const T* wr = sWc + (size_t)(kc & 1) * KC * N3;
#pragma unroll
      for (int k = 0; k < KC; k += 4) {
        T xv[TM][4];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
          for (int u = 0; u < 4; ++u) xv[i][u] = xr[i * XS + k + u];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          T wv[TN];
#pragma unroll
          for (int j = 0; j < TN; ++j) wv[j] = wr[(k + u) * N3 + cg + NCG * j];
#pragma unroll
          for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] = fma(xv[i][u], wv[j], acc[i][j]);
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < TM; ++i) {
      const int r = rg * TM + i;
      const T s = r < rows ? sS[r] : T(0);
#pragma unroll
      for (int j = 0; j < TN; ++j) {
        const int col = cg + NCG * j;
        T v = acc[i][j];
        if (col < GW) v *= s * qscale;
        else if (col < 2 * GW) v *= s;
        sQ[r * QS + col] = v;
      }
    }
    __syncthreads();

    // ---- 2. attention of the group's heads (outputs into the q slots)
    tile_attention<T, HG, D, GW, NT, QS>(sQ, meta, 0, warp, lane, a.smooth ? a.nnei_max : 0);
    __syncthreads();
    // ---- 3. the group's output columns, row by row (coalesced segments)
    constexpr int OV = GW * (int)sizeof(T) / 16;
    for (int e = tid; e < rows * OV; e += NT) {
      const int r = e / OV, v = e - r * OV;
      const int hh = (v * (16 / (int)sizeof(T))) / D;
      const int t0 = v * (16 / (int)sizeof(T)) - hh * D;
      const T* src = sQ + r * QS + hh * D + t0;
      T* dst = out + (row0 + r) * C + g * GW + hh * D + t0;
#pragma unroll
      for (int u = 0; u < 16 / (int)sizeof(T); ++u) dst[u] = src[u];
    }
    __syncthreads();
  }
}

}  // namespace mlg
