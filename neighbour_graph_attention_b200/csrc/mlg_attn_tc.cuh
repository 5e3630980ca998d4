// mlg_attn_tc.cuh -- fp32 block-dense attention whose projection runs on the
// 5th-generation tensor cores (tcgen05.mma kind::tf32, accumulator in TMEM).
//
// Same per-centre attention as mlg_attn_tile.cuh (NeighborGraph issue,
// Proposed fix).  The projection QKV [128 rows][3C] = X [128][C] . W [C][3C]
// of a tile is one UMMA of M = 128, N = 3C per 8-wide K step.  TF32 keeps 10
// mantissa bits, so each operand is split x = hi + lo (both TF32) and the
// product is hi.hi + hi.lo + lo.hi ("3xTF32"), accumulated in fp32 in TMEM:
// the error is that of an fp32 product, not of TF32.
//
// Operands sit in shared memory in the K-major canonical layout without
// swizzle: 8-row x 16-byte core matrices, consecutive 8-row groups 128 bytes
// apart (SBO), consecutive 4-element K chunks ROWS * 16 bytes apart (LBO).
// One elected thread issues the MMAs and commits them to an mbarrier; the
// warps then read the accumulator rows out of TMEM (tcgen05.ld 32x32b), fold
// the switch weights and 1/sqrt(d) into q and k, and run the attention on the
// SIMT units (tile_attention).  The tile's slab arrives by one TMA bulk copy
// and leaves by one bulk copy per row; the split operands and the raw slab
// share the QKV buffer, which is written only after the MMAs completed.
#pragma once

#include <cuda.h>

#include "mlg_common.cuh"
#include "mlg_attn_tile.cuh"

namespace mlg {

// 2-D tiled TMA load of a box {4 floats, 128 rows} at (x, y) into shared memory.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ uint32_t kmajor_offset(int r, int k, int rows) {
  return (uint32_t)(((k >> 2) * (rows >> 3) + (r >> 3)) * 128 + (r & 7) * 16 + (k & 3) * 4);
}

// UMMA shared-memory descriptor: K-major, no swizzle, version 1 (sm_100).
__device__ __forceinline__ uint64_t umma_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}

__device__ __forceinline__ float tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

__device__ __forceinline__ void umma_tf32(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t addr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(addr));
}

__device__ __forceinline__ void tmem_ld8(uint32_t addr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7])
      : "r"(addr));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// The wait, with the 16 registers of one load tied to it, so that the
// compiler cannot read them before the load has landed.
__device__ __forceinline__ void tmem_wait_ld16(uint32_t* v) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15])
               :
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

template <int C, int D, int NT>
struct TcCfg {
  static constexpr int R = 128;                 // tile rows = UMMA M
  static constexpr int N3 = 3 * C;              // UMMA N
  static constexpr int QS = N3 + 4;             // QKV row stride (floats)
  static constexpr int NCOL = N3 <= 128 ? 128 : 256;   // TMEM columns (power of 2)
  static constexpr size_t B_BYTES = (size_t)N3 * C * 4;  // one of B_hi, B_lo
  static constexpr size_t A_BYTES = (size_t)R * C * 4;   // one of A_hi, A_lo
  static constexpr size_t X_BYTES = (size_t)R * C * 4;   // raw slab, K-major order
  static constexpr size_t Q_BYTES = (size_t)R * QS * 4;
  static constexpr size_t REG_BYTES =
      (Q_BYTES > 2 * A_BYTES + X_BYTES ? Q_BYTES : 2 * A_BYTES + X_BYTES);
  static constexpr size_t OFF_BHI = 0;
  static constexpr size_t OFF_BLO = OFF_BHI + B_BYTES;
  static constexpr size_t OFF_REG = (OFF_BLO + B_BYTES + 1023) / 1024 * 1024;
  static constexpr size_t OFF_AHI = OFF_REG;                 // inside the QKV region
  static constexpr size_t OFF_ALO = OFF_AHI + A_BYTES;
  static constexpr size_t OFF_X = OFF_ALO + A_BYTES;
  // a slab buffer of its own (prefetched during the previous tile) when the
  // shared memory allows two CTAs per SM with it
  static constexpr bool PREFETCH = (C <= 32);
  static constexpr size_t OFF_XP = OFF_REG + (REG_BYTES + 1023) / 1024 * 1024;
  static constexpr size_t OFF_S = PREFETCH ? OFF_XP + X_BYTES : OFF_REG + (REG_BYTES + 15) / 16 * 16;
  static constexpr size_t OFF_META = OFF_S + (size_t)R * 4;
  static constexpr size_t OFF_BAR = (OFF_META + sizeof(TileMeta) + 15) / 16 * 16;
  static constexpr size_t SMEM = OFF_BAR + 32;
  static_assert(C % 8 == 0 && N3 % 16 == 0 && N3 <= 256, "UMMA shape");
  static_assert((NT / 32) % 4 == 0, "warps come in groups of 4 (TMEM lane quadrants)");
};

template <int C, int D, int NT>
__global__ void __launch_bounds__(NT) k_attn_tc(TileArgs a, const __grid_constant__ CUtensorMap gmap) {
  using Cfg = TcCfg<C, D, NT>;
  constexpr int R = Cfg::R, N3 = Cfg::N3, QS = Cfg::QS, H = C / D;
  constexpr int NW = NT / 32, NQUART = NW / 4;  // warps per TMEM lane quadrant
  extern __shared__ __align__(1024) unsigned char smem_tc[];
  float* sBhi = reinterpret_cast<float*>(smem_tc + Cfg::OFF_BHI);
  float* sBlo = reinterpret_cast<float*>(smem_tc + Cfg::OFF_BLO);
  float* sQ = reinterpret_cast<float*>(smem_tc + Cfg::OFF_REG);
  char* sAhi = reinterpret_cast<char*>(smem_tc + Cfg::OFF_AHI);
  char* sAlo = reinterpret_cast<char*>(smem_tc + Cfg::OFF_ALO);
  float* sX = reinterpret_cast<float*>(smem_tc + (Cfg::PREFETCH ? Cfg::OFF_XP : Cfg::OFF_X));
  float* sS = reinterpret_cast<float*>(smem_tc + Cfg::OFF_S);
  TileMeta& meta = *reinterpret_cast<TileMeta*>(smem_tc + Cfg::OFF_META);
  uint64_t* bar_x = reinterpret_cast<uint64_t*>(smem_tc + Cfg::OFF_BAR);
  uint64_t* bar_mma = bar_x + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar_x + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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
    mbar_init(bar_x, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tslot)),
                 "r"(Cfg::NCOL));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N3 >> 3) << 17) |
                         ((uint32_t)(R >> 4) << 24);
  const float qscale = (float)(1.4426950408889634 / sqrt((double)D));
  uint32_t ph_x = 0u, ph_mma = 0u;
  int loaded_layer = -1;

  // thread 0: plan the next tile into meta slot b and start its slab copy
  auto plan_and_load = [&](int b) {
      int c = meta.next_c, k = 0, rows = 0, tasks = 0;
      const int c_end = meta.c_end;
      // skip to the next centre this kernel takes, 16 row starts per step so
      // that their loads go out together (with a lower row bound most
      // centres are left to another kernel)
      while (c < c_end) {
        if (c + 16 <= c_end) {
          long long rp[17];
#pragma unroll
          for (int u = 0; u <= 16; ++u) rp[u] = a.row_ptr[c + u];
          int u = 0;
          for (; u < 16; ++u) {
            const int n = (int)(rp[u + 1] - rp[u]);
            if (n > a.min_n && n <= R && n <= a.nnei_max) break;
            if (n > a.nnei_max) atomicOr(a.status, (uint32_t)MLG_STATUS_ROW_TOO_LONG);
          }
          c += u;
          if (u < 16) break;
          continue;
        }
        const int n = (int)(a.row_ptr[c + 1] - a.row_ptr[c]);
        if (n > a.min_n && n <= R && n <= a.nnei_max) break;
        if (n > a.nnei_max) atomicOr(a.status, (uint32_t)MLG_STATUS_ROW_TOO_LONG);
        ++c;
      }
      meta.row0[b] = c < c_end ? a.row_ptr[c] : 0;
      while (c < c_end && k < 64) {
        const int n = (int)(a.row_ptr[c + 1] - a.row_ptr[c]);
        if (n <= a.min_n || n > R || n > a.nnei_max || rows + n > R) break;
        meta.off[b][k] = rows;
        meta.task0[b][k] = tasks;
        tasks += (n * H + 31) / 32;
        rows += n;
        ++k;
        ++c;
      }
      meta.off[b][k] = rows;
      meta.task0[b][k] = tasks;
      meta.ncent[b] = k;
      meta.nrows[b] = rows;
      meta.next_c = c;
      if (rows > 0) {
        // C / 4 tensor loads of {4 columns x 128 rows}: each lands as one
        // K-chunk column of 8-row x 16-byte core matrices (the K-major layout)
        fence_proxy_async();
        mbar_expect_tx(bar_x, (uint32_t)(R * C * 4));
        for (int cc = 0; cc < C / 4; ++cc)
          tma_load_2d(reinterpret_cast<char*>(sX) + cc * R * 16, &gmap, 4 * cc,
                      (int)meta.row0[b], bar_x);
      }
  };

  int cur = 0;
  if (tid == 0) plan_and_load(0);
  while (true) {
    if (tid == 0 && meta.nrows[cur] > 0 && !mbar_wait(bar_x, ph_x)) meta.fail = 1;
    __syncthreads();
    const int rows = meta.nrows[cur];
    const int64_t row0 = meta.row0[cur];
    if (rows == 0 || meta.fail) break;
    ph_x ^= 1u;
    for (int t = tid; t < rows; t += NT) sS[t] = (float)a.sw[row0 + t];

    for (int layer = 0; layer < a.n_layers; ++layer) {
      // ---- weights of the layer: B^T split into TF32 hi / lo, K-major layout
      if (loaded_layer != layer) {
        for (int e = tid; e < C * N3; e += NT) {
          const int k = e / N3, nn = e - k * N3;
          const int m = nn / C, cc = nn - m * C;
          const float w = static_cast<const float*>(a.W[3 * layer + m])[k * C + cc];
          const float hi = tf32_rna(w);
          const uint32_t off = kmajor_offset(nn, k, N3);
          *reinterpret_cast<float*>(reinterpret_cast<char*>(sBhi) + off) = hi;
          *reinterpret_cast<float*>(reinterpret_cast<char*>(sBlo) + off) = tf32_rna(w - hi);
        }
        loaded_layer = layer;
      }
      // ---- the tile's rows split into TF32 hi / lo (rows >= `rows` zero).
      // Layer 0 reads the raw slab, later layers the previous output in the q
      // slots; both lie in the region the split operands occupy, so every
      // thread reads its elements first and writes after a barrier.
      // Element e is the e-th float of the K-major layout (consecutive threads
      // write consecutive words): core matrix e / 32 = (k / 4) * (R / 8) + r / 8,
      // position e % 32 = (r % 8) * 4 + k % 4.
      constexpr int PER = R * C / NT;
      static_assert(PER * NT == R * C, "split work per thread");
      float xin[PER];
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int e = tid + i * NT, core = e >> 5, w = e & 31;
        const int r = (core % (R / 8)) * 8 + (w >> 2), k = (core / (R / 8)) * 4 + (w & 3);
        xin[i] = r < rows ? (layer == 0 ? sX[e] : sQ[r * QS + k]) : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int e = tid + i * NT;
        const float hi = tf32_rna(xin[i]);
        reinterpret_cast<float*>(sAhi)[e] = hi;
        reinterpret_cast<float*>(sAlo)[e] = tf32_rna(xin[i] - hi);
      }
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
      // the slab buffer is free: with its own buffer, the next tile's copy
      // starts now and lands while this tile computes
      if (Cfg::PREFETCH && layer == a.n_layers - 1 && tid == 0) plan_and_load(cur ^ 1);
      // ---- 1. the projection on the tensor cores (one elected thread)
      if (tid == 0) {
        tc_fence_after();
        const uint32_t ahi = smem_u32(sAhi), alo = smem_u32(sAlo);
        const uint32_t bhi = smem_u32(sBhi), blo = smem_u32(sBlo);
#pragma unroll
        for (int s = 0; s < C / 8; ++s) {
          const uint32_t aoff = (uint32_t)(s * R * 32), boff = (uint32_t)(s * N3 * 32);
          const uint64_t dah = umma_sdesc(ahi + aoff, R * 16, 128);
          const uint64_t dal = umma_sdesc(alo + aoff, R * 16, 128);
          const uint64_t dbh = umma_sdesc(bhi + boff, N3 * 16, 128);
          const uint64_t dbl = umma_sdesc(blo + boff, N3 * 16, 128);
          umma_tf32(tmem, dal, dbh, idesc, s > 0 ? 1u : 0u);  // small terms first
          umma_tf32(tmem, dah, dbl, idesc, 1u);
          umma_tf32(tmem, dah, dbh, idesc, 1u);
        }
        umma_commit(bar_mma);
        if (!mbar_wait(bar_mma, ph_mma)) meta.fail = 1;
      }
      __syncthreads();
      ph_mma ^= 1u;
      if (meta.fail) break;
      tc_fence_after();
      // ---- TMEM -> QKV rows (the split operands are dead now), scaled
      {
        const int quad = warp & 3, part = warp >> 2;   // lane quadrant, column part
        const int row = quad * 32 + lane;
        const float s = row < rows ? sS[row] : 0.f;
        constexpr int CPW = N3 / NQUART;               // columns per warp
        static_assert(CPW % 8 == 0, "8-column loads");
#pragma unroll
        for (int c0 = 0; c0 < CPW; c0 += 8) {
          const int col0 = part * CPW + c0;
          uint32_t v[8];
          tmem_ld8(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)col0, v);
          tmem_wait_ld();
          // 8 columns never straddle q / k / v (C is a multiple of 8)
          const float f = col0 < C ? s * qscale : (col0 < 2 * C ? s : 1.f);
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
      // ---- 2. attention (SIMT), output into the q slots
      tile_attention<float, H, D, C, NT, QS>(sQ, meta, cur, warp, lane,
                                             a.smooth ? a.nnei_max : 0);
      __syncthreads();
    }
    if (meta.fail) break;
    // ---- 3. write back: one bulk copy per row from the q slots
    fence_proxy_async();
    __syncthreads();
    if (warp == 0) {
      for (int r = lane; r < rows; r += 32)
        bulk_s2g(out + (row0 + r) * C, sQ + r * QS, (uint32_t)(C * 4));
      bulk_commit();
      bulk_wait_read_all();  // (without a slab buffer of its own, the next slab lands here)
    }
    __syncthreads();
    if (Cfg::PREFETCH) {
      cur ^= 1;
    } else if (tid == 0) {
      plan_and_load(cur);
    }
  }
  if (warp == 0) bulk_wait_all();
  if (tid == 0 && meta.fail) {
    atomicOr(a.status, kStatusTimeout);
    // a prefetched slab may still be landing: let it finish before exit
    if (Cfg::PREFETCH) mbar_wait(bar_x, ph_x);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(Cfg::NCOL));
  }
}

}  // namespace mlg
