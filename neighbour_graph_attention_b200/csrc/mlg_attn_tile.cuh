// mlg_attn_tile.cuh -- fused multi-layer block-dense attention for channel
// counts whose three projection matrices fit in shared memory (sm_100a).
//
// NeighborGraph issue ("NeighborGraph attention is 4-9x slower than dense and
// OOM-prone"), Proposed fix: per centre, gather the compact block of its edge
// features through destination_row_ptr, run dense attention with per-row
// masks, write back to the edge axis.  Because the edges of a centre are one
// contiguous CSR slab, a tile of consecutive centres is one contiguous
// [rows][C] slab of G: it is moved global->shared and shared->global by TMA
// bulk copies (cp.async.bulk, no multicast).  A centre's output rows depend
// only on its own input rows, so every layer of the stack runs on the
// resident tile before it is written back (G^{l+1} = O^l never leaves the SM).
//
// Per tile and layer:
//   1. QKV = X [rows][C] . [Wq | Wk | Wv] [C][3C]: register-tiled FMA GEMM
//      from shared memory; the epilogue folds s_a / sqrt(d) into q (times
//      log2 e for fp32, whose softmax uses exp2) and s_b into k.
//   2. attention: one lane per (query row a, head h) of a centre, lanes of a
//      warp in lock-step over key rows b, so k_b and v_b are broadcast
//      shared-memory reads; softmax with a running max in blocks of 8 keys.
//   3. O overwrites X in shared memory; the next layer's weights stream in
//      (TMA) while the attention runs.
// Persistent CTAs: CTA b owns the centres whose first edge row lies in the
// b-th equal share of the E rows; it packs consecutive centres into tiles of
// at most R rows and prefetches the next tile's slab.  Centres with more than
// R edges are left to the generic kernel (mlg_attn.cuh).
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

// Bounded wait (about a second at most): false if the phase never completed.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (int it = 0; it < (1 << 22); ++it) {
    if (mbar_test(bar, parity)) return true;
    if (it > 64) __nanosleep(200);
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

// ---------------------------------------------------------------- the kernel

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

template <typename T, int C, int D, int R, int NT, int TM, int TN, int XB>
struct TileCfg {
  static constexpr int H = C / D;
  static constexpr int N3 = 3 * C;              // GEMM output columns
  static constexpr int NCG = N3 / TN;           // column groups
  static constexpr int NRG = R / TM;            // row groups
  static constexpr int QS = N3 + (sizeof(T) == 8 ? 1 : 4);  // QKV row stride (elements)
  static constexpr int MAXC = 64;               // centres per tile (bookkeeping arrays)
  static_assert(NCG * NRG == NT, "thread grid must cover the tile");
  static_assert(C % D == 0 && D % 4 == 0, "head size");
  static_assert(C % NCG == 0, "column groups must not straddle q/k/v");
  // shared memory layout (bytes)
  static constexpr size_t X_BYTES = (size_t)R * C * sizeof(T);
  static constexpr size_t W_BYTES = (size_t)3 * C * C * sizeof(T);
  static constexpr size_t Q_BYTES = (size_t)R * QS * sizeof(T);
  static_assert(XB == 1 || XB == 2, "one or two tile buffers");
  static constexpr size_t OFF_X0 = 0;
  static constexpr size_t OFF_X1 = OFF_X0 + X_BYTES;
  static constexpr size_t OFF_W = OFF_X0 + XB * X_BYTES;
  static constexpr size_t OFF_Q = OFF_W + W_BYTES;
  static constexpr size_t OFF_S = OFF_Q + Q_BYTES;
  static constexpr size_t OFF_META = (OFF_S + (size_t)R * sizeof(T) + 15) / 16 * 16;
  static constexpr size_t SMEM = OFF_META + sizeof(TileMeta);
};



// One key block of the running-max softmax for one lane (query row, head):
// logits of keys [b0, b0 + 8) (masked to -inf at and beyond n when TAIL),
// rescale of the running sum and output when the block raises the maximum,
// then accumulation of exp(l - max) v.  fp32 logits are in log2 units (q
// carries log2 e), fp64 ones in natural units.
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
template <typename T, int HEADS, int D, int KOFF, int NT, int QS>
__device__ __forceinline__ void tile_attention(T* sQ, const TileMeta& meta, int buf, int warp,
                                               int lane) {
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

template <typename T, int C, int D, int R, int NT, int TM, int TN, int XB>
__global__ void __launch_bounds__(NT) k_attn_tile(TileArgs a) {
  using Cfg = TileCfg<T, C, D, R, NT, TM, TN, XB>;
  constexpr int H = Cfg::H, NCG = Cfg::NCG, QS = Cfg::QS;
  extern __shared__ __align__(128) unsigned char smem[];
  T* sX[2] = {reinterpret_cast<T*>(smem + Cfg::OFF_X0),
              reinterpret_cast<T*>(smem + (XB == 2 ? Cfg::OFF_X1 : Cfg::OFF_X0))};
  T* sW = reinterpret_cast<T*>(smem + Cfg::OFF_W);
  T* sQ = reinterpret_cast<T*>(smem + Cfg::OFF_Q);
  T* sS = reinterpret_cast<T*>(smem + Cfg::OFF_S);
  TileMeta& meta = *reinterpret_cast<TileMeta*>(smem + Cfg::OFF_META);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const T* G = static_cast<const T*>(a.G);
  T* out = static_cast<T*>(a.out);
  const int64_t E = a.row_ptr[a.n_centres];
  if (E > a.capacity || (*a.status & MLG_STATUS_CAPACITY)) return;

  // ---- set-up: my centre range, barriers, first weights, first tile
  if (tid == 0) {
    const int64_t r0 = E * blockIdx.x / gridDim.x, r1 = E * (blockIdx.x + 1) / gridDim.x;
    // first centre whose first row is >= r (lower bound over row_ptr[0..n_centres))
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
    mbar_init(&meta.bar_x[0], 1);
    mbar_init(&meta.bar_x[1], 1);
    mbar_init(&meta.bar_w, 1);
    fence_mbar_init();
  }
  __syncthreads();

  // thread 0: pack the next tile (consecutive centres, <= R rows, skipping
  // centres with more than R edges) into buffer b and start its slab copy
  auto plan_and_load = [&](int b) {
    int c = meta.next_c, k = 0, rows = 0;
    const int c_end = meta.c_end;
    // skip leading empty or oversized centres
    while (c < c_end) {
      int n = (int)(a.row_ptr[c + 1] - a.row_ptr[c]);
      if (n > 0 && n <= R) break;
      ++c;
    }
    meta.c0[b] = c;
    meta.row0[b] = c < c_end ? a.row_ptr[c] : 0;
    int tasks = 0;
    while (c < c_end && k < Cfg::MAXC) {
      int n = (int)(a.row_ptr[c + 1] - a.row_ptr[c]);
      if (n > R) break;                 // oversized: ends the tile (handled elsewhere)
      if (rows + n > R) break;
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
      fence_proxy_async();
      uint32_t bytes = (uint32_t)(rows * C * sizeof(T));
      mbar_expect_tx(&meta.bar_x[b], bytes);
      bulk_g2s(sX[b], G + meta.row0[b] * C, bytes, &meta.bar_x[b]);
    }
  };

  auto load_weights = [&](int layer) {
    fence_proxy_async();
    const uint32_t bytes = (uint32_t)(C * C * sizeof(T));
    mbar_expect_tx(&meta.bar_w, 3 * bytes);
#pragma unroll
    for (int m = 0; m < 3; ++m) bulk_g2s(sW + m * C * C, a.W[3 * layer + m], bytes, &meta.bar_w);
  };

  if (tid == 0) {
    plan_and_load(0);
    if (meta.nrows[0] > 0) load_weights(0);  // a CTA without tiles starts no copy
  }
  __syncthreads();

  uint32_t ph_x[2] = {0u, 0u}, ph_w = 0u;
  const T qscale = sizeof(T) == 4 ? T(1.4426950408889634 / sqrt((double)D))
                                  : T(1.0 / sqrt((double)D));
  int buf = 0;
  bool weights_pending = meta.nrows[0] > 0;

  while (true) {
    if (meta.nrows[buf] == 0) break;  // uniform: written by thread 0 before a barrier
    if (tid == 0) {
      if (XB == 2) {
        // prefetch the next tile into the other buffer (its last store must be read out)
        bulk_wait_read_all();
        plan_and_load(buf ^ 1);
      }
      bool okx = mbar_wait(&meta.bar_x[buf], ph_x[buf]);
      if (!okx) meta.fail = 1;
    }
    __syncthreads();
    if (meta.fail) break;
    ph_x[buf] ^= 1u;
    const int rows = meta.nrows[buf], ncent = meta.ncent[buf];
    const int64_t row0 = meta.row0[buf];
    for (int t = tid; t < rows; t += NT) sS[t] = (T)a.sw[row0 + t];
    T* X = sX[buf];

    for (int layer = 0; layer < a.n_layers; ++layer) {
      if (weights_pending) {
        if (tid == 0 && !mbar_wait(&meta.bar_w, ph_w)) meta.fail = 1;
        ph_w ^= 1u;
        weights_pending = false;
      }
      __syncthreads();
      if (meta.fail) break;

      // ---- 1. QKV = X . W (rows >= `rows` of X hold stale data; their outputs are unused)
      {
        const int rg = tid / NCG, cg = tid % NCG;
        T acc[TM][TN];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
          for (int j = 0; j < TN; ++j) acc[i][j] = T(0);
        const T* xr = X + (rg * TM) * C;
#pragma unroll 2
        for (int k = 0; k < C; k += 4) {
          T xv[TM][4];
#pragma unroll
          for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int u = 0; u < 4; ++u) xv[i][u] = xr[i * C + k + u];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            T wv[TN];
#pragma unroll
            for (int j = 0; j < TN; ++j) {
              const int col = cg + NCG * j;
              const int m = col / C, cc = col - m * C;
              wv[j] = sW[m * C * C + (k + u) * C + cc];
            }
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
              for (int j = 0; j < TN; ++j) acc[i][j] = fma(xv[i][u], wv[j], acc[i][j]);
          }
        }
#pragma unroll
        for (int i = 0; i < TM; ++i) {
          const int r = rg * TM + i;
          const T s = r < rows ? sS[r] : T(0);
#pragma unroll
          for (int j = 0; j < TN; ++j) {
            const int col = cg + NCG * j;
            T v = acc[i][j];
            if (col < C) v *= s * qscale;
            else if (col < 2 * C) v *= s;
            sQ[r * QS + col] = v;
          }
        }
      }
      __syncthreads();
      // the next layer's weights stream in while the attention runs
      // (with one buffer the next tile is not planned yet: any centre left may start one)
      const bool more = layer + 1 < a.n_layers ||
                        (XB == 2 ? meta.nrows[buf ^ 1] > 0 : meta.next_c < meta.c_end);
      if (a.n_layers > 1 && tid == 0 && more) load_weights((layer + 1) % a.n_layers);
      if (a.n_layers > 1) weights_pending = more;

      // ---- 2. attention: warp tasks of 32 (head, row) pairs of one centre
      tile_attention<T, C / D, D, C, NT, QS>(sQ, meta, buf, warp, lane);
      __syncthreads();
      for (int e = tid; e < rows * C; e += NT) {
        const int r = e / C, col = e - r * C;
        X[e] = sQ[r * QS + col];
      }
      __syncthreads();
    }
    if (meta.fail) break;
    // ---- 3. write the tile back: one bulk copy of the contiguous slab
    fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
      bulk_s2g(out + row0 * C, X, (uint32_t)(rows * C * sizeof(T)));
      bulk_commit();
      if (XB == 1) {
        bulk_wait_read_all();
        plan_and_load(0);
      }
    }
    if (XB == 2) buf ^= 1;
    __syncthreads();
  }
  if (tid == 0) {
    bulk_wait_all();
    if (meta.fail) {
      atomicOr(a.status, kStatusTimeout);
      // let copies in flight land before the CTA's shared memory is released
      mbar_wait(&meta.bar_x[buf ^ 1], ph_x[buf ^ 1]);
      mbar_wait(&meta.bar_w, ph_w);
    } else if (weights_pending) {
      mbar_wait(&meta.bar_w, ph_w);  // never left in flight at exit
    }
  }
}

}  // namespace mlg
