// mlg_attn_tile.cuh -- pieces shared by the fused block-dense attention
// kernels (sm_100a): the tile arguments and plan, PTX helpers for mbarriers
// and TMA bulk copies, and the per-centre attention loop over a resident tile.
//
// NeighborGraph issue ("NeighborGraph attention is 4-9x slower than dense and
// OOM-prone"), Proposed fix: per centre, gather the compact block of its edge
// features through destination_row_ptr, run dense attention with per-row
// masks, write back to the edge axis.  Because the edges of a centre are one
// contiguous CSR slab, a tile of consecutive centres is one contiguous
// [rows][C] slab of G; a centre's output rows depend only on its own input
// rows, so every layer of a stack can run on the resident tile before it is
// written back (G^{l+1} = O^l never leaves the SM).
//
// tile_attention(): one lane per (query row a, head h) of a centre, the lanes
// of a warp in lock-step over key rows b, so k_b and v_b are broadcast
// shared-memory reads; softmax with a running max in blocks of 8 keys.  Used
// by the tcgen05 kernel (mlg_attn_tc.cuh) and the head-group kernel
// (mlg_attn_hg.cuh).
#pragma once

#include "mlg_common.cuh"

namespace mlg {

constexpr uint32_t kStatusTimeout = 64u;  // an mbarrier wait ran out (never expected)

constexpr int kMaxFusedLayers = 32;

struct TileArgs {
  const int64_t* row_ptr;
  const double* sw;
  int64_t n_centres;
  int64_t capacity;
  int n_layers;  // 1 .. kMaxFusedLayers
  int nnei_max;  // centres with more edges are skipped and flagged (MLG_STATUS_ROW_TOO_LONG)
  int min_n;     // centres with at most min_n edges are left to another kernel (0: none)
  int smooth;    // slot-occupancy softmax: nnei_max - n phantom slots of logit 0, value 0
  const void* G;
  void* out;
  const void* W[3 * kMaxFusedLayers];  // q, k, v of each layer: device [C][C]
  uint32_t* status;
};

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// One potentially blocking test: the hardware may hold the thread (without
// issuing) until the phase completes or a system-dependent time limit passes.
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait: false if the phase has not completed after about a second
// (global timer) or 2^24 tests, whichever comes first.  A waiting warp is
// held by try_wait rather than spinning, so it takes no issue slots from the
// warps that work.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (int it = 0; it < (1 << 24); ++it) {
    if (mbar_try(bar, parity)) return true;
    if (globaltimer_ns() - t0 > 1000000000ull) return false;
  }
  return false;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_s2g(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

template <typename T>
__device__ __forceinline__ T softmax_exp(T x);
template <>
__device__ __forceinline__ float softmax_exp<float>(float x) { return exp2f(x); }
template <>
__device__ __forceinline__ double softmax_exp<double>(double x) { return exp(x); }

// ---------------------------------------------------------------- tiles

struct TileMeta {
  uint64_t bar_x[2];
  uint64_t bar_w;
  int64_t row0[2];      // first global row of the tile in each buffer
  int nrows[2];
  int ncent[2];
  int c0[2];            // first centre of the tile in each buffer
  int off[2][65];       // local row offset of each centre, off[ncent] = nrows (<= 64 centres)
  int task0[2][65];     // first warp task of each centre
  int next_c;           // first centre not yet assigned to a tile
  int c_end;
  int fail;
};

template <typename T, int D, bool TAIL>
__device__ __forceinline__ void softmax_block(const T* q, T* o, T& mx, T& l, const T* kb,
                                              const T* vb, int b0, int n, int QS) {
  T s[8];
  T bm = T(-INFINITY);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int b = b0 + j;
    T acc = T(0);
    if (!TAIL || b < n) {
      const T* kr = kb + b * QS;
      if constexpr (sizeof(T) == 4 && D % 4 == 0) {
        // 16-byte broadcast loads, packed fp32x2 FMAs
        float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int t = 0; t < D; t += 4) {
          const float4 k4 = *reinterpret_cast<const float4*>(kr + t);
          a2 = __ffma2_rn(make_float2(q[t], q[t + 1]), make_float2(k4.x, k4.y), a2);
          a2 = __ffma2_rn(make_float2(q[t + 2], q[t + 3]), make_float2(k4.z, k4.w), a2);
        }
        acc = a2.x + a2.y;
      } else {
#pragma unroll
        for (int t = 0; t < D; ++t) acc = fma(q[t], kr[t], acc);
      }
    } else {
      acc = T(-INFINITY);
    }
    s[j] = acc;
    bm = bm > acc ? bm : acc;
  }
  if (bm > mx) {
    const T sc = softmax_exp<T>(mx - bm);  // exp(-inf) = 0 on the first block
    l *= sc;
#pragma unroll
    for (int t = 0; t < D; ++t) o[t] *= sc;
    mx = bm;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int b = b0 + j;
    if (!TAIL || b < n) {
      const T pj = softmax_exp<T>(s[j] - mx);
      l += pj;
      const T* vr = vb + b * QS;
      if constexpr (sizeof(T) == 4 && D % 4 == 0) {
        const float2 p2 = make_float2(pj, pj);
#pragma unroll
        for (int t = 0; t < D; t += 4) {
          const float4 v4 = *reinterpret_cast<const float4*>(vr + t);
          float2 o2 = __ffma2_rn(p2, make_float2(v4.x, v4.y), make_float2(o[t], o[t + 1]));
          float2 o3 = __ffma2_rn(p2, make_float2(v4.z, v4.w), make_float2(o[t + 2], o[t + 3]));
          o[t] = o2.x;
          o[t + 1] = o2.y;
          o[t + 2] = o3.x;
          o[t + 3] = o3.y;
        }
      } else {
#pragma unroll
        for (int t = 0; t < D; ++t) o[t] = fma(pj, vr[t], o[t]);
      }
    }
  }
}

// Attention of one tile from its QKV rows in shared memory [rows][QS]: head h
// of the HEADS handled here has q at column h d, k at KOFF + h d and v at
// 2 KOFF + h d; q carries s_a / sqrt(d) (times log2 e in fp32), k carries s_b.
// Warp tasks: 32 consecutive (head, row) pairs of one centre; lanes of a warp
// walk the keys in lock-step, so k_b and v_b are broadcast reads.  The output
// of (row, h) overwrites the q slot that only its own lane read.
// With smooth_nnei > 0 (the slot-occupancy softmax, NeighborGraph issue,
// Numerics note) a centre of n edges also has phi = smooth_nnei - n phantom
// slots of logit 0 and value 0; they enter the running softmax as a first
// block: maximum 0, sum phi, output 0.
template <typename T, int HEADS, int D, int KOFF, int NT, int QS>
__device__ __forceinline__ void tile_attention(T* sQ, const TileMeta& meta, int buf, int warp,
                                               int lane, int smooth_nnei = 0) {
  const int ncent = meta.ncent[buf];
  const int ntask = meta.task0[buf][ncent];
  for (int task = warp; task < ntask; task += NT / 32) {
    int ci = 0;
    while (meta.task0[buf][ci + 1] <= task) ++ci;
    const int base = meta.off[buf][ci];
    const int n = meta.off[buf][ci + 1] - base;
    const int p = (task - meta.task0[buf][ci]) * 32 + lane;
    const bool valid = p < n * HEADS;
    const int h = valid ? p / n : 0;
    const int row = valid ? p - h * n : 0;
    T q[D], o[D];
    const T* qrow = sQ + (base + row) * QS + h * D;
#pragma unroll
    for (int t = 0; t < D; ++t) {
      q[t] = qrow[t];
      o[t] = T(0);
    }
    T mx = T(-INFINITY), l = T(0);
    if (smooth_nnei > n) {
      mx = T(0);
      l = T(smooth_nnei - n);
    }
    const T* kb = sQ + base * QS + KOFF + h * D;
    const T* vb = sQ + base * QS + 2 * KOFF + h * D;
    const int nfull = n & ~7;
    for (int b0 = 0; b0 < nfull; b0 += 8)
      softmax_block<T, D, false>(q, o, mx, l, kb, vb, b0, n, QS);
    if (nfull < n) softmax_block<T, D, true>(q, o, mx, l, kb, vb, nfull, n, QS);
    if (valid) {
      // this lane alone read the q slot of (row, h): reuse it for the output
      // (the padded QKV stride spreads rows over banks; X's stride would not)
      const T rl = T(1) / l;
      T* qo = sQ + (base + row) * QS + h * D;
#pragma unroll
      for (int t = 0; t < D; ++t) qo[t] = o[t] * rl;
    }
  }
}

}  // namespace mlg
