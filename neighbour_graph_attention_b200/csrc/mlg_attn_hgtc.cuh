// mlg_attn_hgtc.cuh -- fp32 block-dense attention for wide features (128
// channels, 8 heads of 16) with the projection on the 5th-generation tensor
// cores (tcgen05.mma kind::tf32, 3xTF32, accumulator in TMEM).
//
// Same per-centre attention as mlg_attn_tile.cuh (NeighborGraph issue,
// Proposed fix).  At 128 channels the projections are most of the work
// (6 n c^2 of the 6 n c^2 + 4 n^2 c flops of a centre), so they go to the
// tensor cores; the per-centre logits and P.V (K = d = 16) stay on the FP32
// pipe (tile_attention).
//
// Grid (centre ranges x head groups): a CTA computes the q, k, v columns of
// two heads, QKV[128 x 96] = X[128 x 128] . W_g[128 x 96], for tiles of
// consecutive centres of at most 128 rows.  W_g (split into TF32 hi / lo,
// 96 KB) stays in shared memory for the whole launch; X streams in four
// K-chunks of 32 channels, each by 2-D TMA boxes of {4 x 128} into the
// K-major core-matrix layout, split into hi / lo and multiplied while the
// next chunk lands.  One layer per launch.
#pragma once

#include <cuda.h>

#include "mlg_common.cuh"
#include "mlg_attn_tile.cuh"
#include "mlg_attn_tc.cuh"

namespace mlg {

namespace hgtc {

constexpr int C = 128, D = 16, HG = 2, GW = HG * D, N3 = 3 * GW, R = 128, KC = 32;
constexpr int NK = C / KC;       // K-chunks
constexpr int NT = 256;
constexpr int NG = (C / D) / HG; // head groups (grid.y)
constexpr int QS = N3 + 4;       // QKV staging row stride (floats)

constexpr size_t W_BYTES = (size_t)N3 * C * 4;    // one of W hi / lo
constexpr size_t X_BYTES = (size_t)R * KC * 4;    // one raw chunk, or one of A hi / lo
constexpr size_t OFF_WHI = 0;
constexpr size_t OFF_WLO = OFF_WHI + W_BYTES;
constexpr size_t OFF_X = OFF_WLO + W_BYTES;       // raw chunks [2]
constexpr size_t OFF_A = OFF_X + 2 * X_BYTES;     // [buffer][hi, lo]
constexpr size_t OFF_Q = OFF_A;                   // QKV staging, after the last MMA
constexpr size_t OFF_S = OFF_A + 4 * X_BYTES;
constexpr size_t OFF_META = OFF_S + (size_t)R * 4;
constexpr size_t OFF_BAR = (OFF_META + sizeof(TileMeta) + 15) / 16 * 16;
constexpr size_t SMEM = OFF_BAR + 48;
static_assert((size_t)R * QS * 4 <= 4 * X_BYTES, "QKV staging fits the A buffers");
static_assert(SMEM <= 227 * 1024, "shared memory");

}  // namespace hgtc

struct HgtcArgs {
  const int64_t* row_ptr;
  const double* sw;
  int64_t n_centres;
  int64_t capacity;
  int nnei_max;
  int smooth;
  void* out;
  const void* Wq;
  const void* Wk;
  const void* Wv;
  uint32_t* status;
};

__global__ void __launch_bounds__(hgtc::NT, 1)
    k_attn_hgtc(HgtcArgs a, const __grid_constant__ CUtensorMap gmap) {
  using namespace hgtc;
  extern __shared__ __align__(1024) unsigned char smem_hg[];
  unsigned char* sm = smem_hg;
  float* sQ = reinterpret_cast<float*>(sm + OFF_Q);
  float* sS = reinterpret_cast<float*>(sm + OFF_S);
  TileMeta& meta = *reinterpret_cast<TileMeta*>(sm + OFF_META);
  uint64_t* bar_x = reinterpret_cast<uint64_t*>(sm + OFF_BAR);     // [2]
  uint64_t* bar_mma = bar_x + 2;                                   // [2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar_x + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y;
  float* out = static_cast<float*>(a.out);
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
    meta.fail = 0;
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar_x[b], 1);
      mbar_init(&bar_mma[b], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tslot)),
                 "r"(128));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // the head group's weights, split into TF32 hi / lo, B operand [96 x 128] K-major
  {
    const float* Wm[3] = {static_cast<const float*>(a.Wq), static_cast<const float*>(a.Wk),
                          static_cast<const float*>(a.Wv)};
    for (int e = tid; e < C * N3; e += NT) {
      const int k = e / N3, nn = e - k * N3;
      const int m = nn / GW, cc = nn - m * GW;
      const float w = Wm[m][(size_t)k * C + g * GW + cc];
      const float hi = tf32_rna(w);
      const uint32_t off = kmajor_offset(nn, k, N3);
      *reinterpret_cast<float*>(sm + OFF_WHI + off) = hi;
      *reinterpret_cast<float*>(sm + OFF_WLO + off) = tf32_rna(w - hi);
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N3 >> 3) << 17) |
                         ((uint32_t)(R >> 4) << 24);
  const float qscale = (float)(1.4426950408889634 / 4.0);  // log2(e) / sqrt(16)
  const int nlim = a.nnei_max < R ? a.nnei_max : R;
  uint32_t ph_x[2] = {0u, 0u}, ph_m[2] = {0u, 0u};

  // thread 0: plan the next tile into meta slot b
  auto plan = [&](int b) {
    int c = meta.next_c, k = 0, rows = 0, tasks = 0;
    const int c_end = meta.c_end;
    while (c < c_end) {
      const int n = (int)(a.row_ptr[c + 1] - a.row_ptr[c]);
      if (n > 0 && n <= nlim) break;
      if (n > a.nnei_max && g == 0) atomicOr(a.status, (uint32_t)MLG_STATUS_ROW_TOO_LONG);
      ++c;
    }
    meta.row0[b] = c < c_end ? a.row_ptr[c] : 0;
    while (c < c_end && k < 64) {
      const int n = (int)(a.row_ptr[c + 1] - a.row_ptr[c]);
      if (n < 1 || n > nlim || rows + n > R) break;
      meta.off[b][k] = rows;
      meta.task0[b][k] = tasks;
      tasks += (n * HG + 31) / 32;
      rows += n;
      ++k;
      ++c;
    }
    meta.off[b][k] = rows;
    meta.task0[b][k] = tasks;
    meta.ncent[b] = k;
    meta.nrows[b] = rows;
    meta.next_c = c;
  };
  // thread 0: K-chunk kc of tile slot b into raw buffer kc & 1
  auto load_chunk = [&](int b, int kc) {
    uint64_t* bar = &bar_x[kc & 1];
    mbar_expect_tx(bar, (uint32_t)X_BYTES);
    for (int cc = 0; cc < KC / 4; ++cc)
      tma_load_2d(sm + OFF_X + (size_t)(kc & 1) * X_BYTES + (size_t)cc * (R * 16), &gmap,
                  KC * kc + 4 * cc, (int)meta.row0[b], bar);
  };

  int cur = 0;
  if (tid == 0) {
    plan(0);
    if (meta.nrows[0] > 0) {
      fence_proxy_async();
      load_chunk(0, 0);
      load_chunk(0, 1);
    }
  }
  __syncthreads();
  while (true) {
    const int rows = meta.nrows[cur];
    const int64_t row0 = meta.row0[cur];
    if (rows == 0 || meta.fail) break;
    for (int t = tid; t < rows; t += NT) sS[t] = (float)a.sw[row0 + t];
    // ---- 1. the projection over four K-chunks on the tensor cores
    for (int kc = 0; kc < NK; ++kc) {
      const int b = kc & 1;
      if (tid == 0) {
        if (!mbar_wait(&bar_x[b], ph_x[b])) meta.fail = 1;
        ph_x[b] ^= 1u;
        if (kc >= 2) {  // the MMAs of chunk kc - 2 have read A buffer b
          if (!mbar_wait(&bar_mma[b], ph_m[b])) meta.fail = 1;
          ph_m[b] ^= 1u;
        }
      }
      __syncthreads();
      if (meta.fail) break;
      // split the raw chunk into A buffer b (rows past the tile are zero)
      const float* sX = reinterpret_cast<const float*>(sm + OFF_X + (size_t)b * X_BYTES);
      float* sAh = reinterpret_cast<float*>(sm + OFF_A + (size_t)(2 * b) * X_BYTES);
      float* sAl = reinterpret_cast<float*>(sm + OFF_A + (size_t)(2 * b + 1) * X_BYTES);
      for (int e = tid; e < R * KC; e += NT) {
        const int core = e >> 5, w = e & 31;
        const int r = (core % (R / 8)) * 8 + (w >> 2);
        const float x = r < rows ? sX[e] : 0.f;
        const float hi = tf32_rna(x);
        sAh[e] = hi;
        sAl[e] = tf32_rna(x - hi);
      }
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        // the raw buffer is free again: the chunk after next lands in it
        if (kc + 2 < NK) load_chunk(cur, kc + 2);
        tc_fence_after();
        const uint32_t ahi = smem_u32(sAh), alo = smem_u32(sAl);
        const uint32_t bhi = smem_u32(sm + OFF_WHI), blo = smem_u32(sm + OFF_WLO);
#pragma unroll
        for (int s = 0; s < KC / 8; ++s) {
          const uint32_t aoff = (uint32_t)(s * R * 32);
          const uint32_t boff = (uint32_t)((KC * kc / 4 + 2 * s) * N3 * 16);
          const uint64_t dah = umma_sdesc(ahi + aoff, R * 16, 128);
          const uint64_t dal = umma_sdesc(alo + aoff, R * 16, 128);
          const uint64_t dbh = umma_sdesc(bhi + boff, N3 * 16, 128);
          const uint64_t dbl = umma_sdesc(blo + boff, N3 * 16, 128);
          const uint32_t acc0 = (kc > 0 || s > 0) ? 1u : 0u;
          umma_tf32(tmem, dal, dbh, idesc, acc0);  // small terms first
          umma_tf32(tmem, dah, dbl, idesc, 1u);
          umma_tf32(tmem, dah, dbh, idesc, 1u);
        }
        umma_commit(&bar_mma[b]);
      }
    }
    if (tid == 0 && !meta.fail) {
      // the last two commits: every MMA of the tile is complete
      for (int b = 0; b < 2; ++b) {
        if (!mbar_wait(&bar_mma[b], ph_m[b])) meta.fail = 1;
        ph_m[b] ^= 1u;
      }
    }
    __syncthreads();
    if (meta.fail) break;
    tc_fence_after();
    // ---- 2. TMEM -> QKV staging (over the A buffers, now unused), scaled
    {
      const int quad = warp & 3, part = warp >> 2;  // lane quadrant, column half
      const int row = quad * 32 + lane;
      const float s = row < rows ? sS[row] : 0.f;
#pragma unroll
      for (int c0 = 0; c0 < N3 / 2; c0 += 8) {
        const int col0 = part * (N3 / 2) + c0;
        uint32_t v[8];
        tmem_ld8(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)col0, v);
        tmem_wait_ld();
        const float f = col0 < GW ? s * qscale : (col0 < 2 * GW ? s : 1.f);
#pragma unroll
        for (int j = 0; j < 8; j += 4) {
          const float4 x4 = make_float4(__uint_as_float(v[j]) * f, __uint_as_float(v[j + 1]) * f,
                                        __uint_as_float(v[j + 2]) * f,
                                        __uint_as_float(v[j + 3]) * f);
          *reinterpret_cast<float4*>(sQ + row * QS + col0 + j) = x4;
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    // the next tile's first two chunks land during the attention (the raw
    // buffers do not overlap the staging)
    if (tid == 0) {
      plan(cur ^ 1);
      if (meta.nrows[cur ^ 1] > 0) {
        fence_proxy_async();
        load_chunk(cur ^ 1, 0);
        load_chunk(cur ^ 1, 1);
      }
    }
    // ---- 3. attention of the group's two heads (outputs into the q slots)
    tile_attention<float, HG, D, GW, NT, QS>(sQ, meta, cur, warp, lane,
                                             a.smooth ? a.nnei_max : 0);
    __syncthreads();
    // ---- 4. the group's output columns, row by row (16-byte pieces)
    for (int e = tid; e < rows * (GW / 4); e += NT) {
      const int r = e / (GW / 4), v = e - r * (GW / 4);
      const float4 x4 = *reinterpret_cast<const float4*>(sQ + r * QS + 4 * v);
      *reinterpret_cast<float4*>(out + (row0 + r) * C + g * GW + 4 * v) = x4;
    }
    __syncthreads();
    cur ^= 1;
  }
  if (tid == 0 && meta.fail) {
    atomicOr(a.status, kStatusTimeout);
    // chunk copies may still be landing: let them finish (bounded)
    mbar_wait(&bar_x[0], ph_x[0]);
    mbar_wait(&bar_x[1], ph_x[1]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128));
  }
}

}  // namespace mlg
