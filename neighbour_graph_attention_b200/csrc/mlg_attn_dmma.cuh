// mlg_attn_dmma.cuh -- fused multi-layer block-dense attention in fp64 on the
// FP64 tensor pipe (mma.sync m8n8k4 .f64, sm_100a).
//
// The per-centre attention of the NeighborGraph issue (Proposed fix: dense
// attention per centre with masks for the ragged tail, written back to the
// edge axis), for c = 32 channels, 4 heads of d = 8, in fp64.  Every product
// is an 8x8x4 fp64 MMA (one instruction per 256 FMAs, at the FP64 FMA rate):
//   projection  QKV [rows][96] = X [rows][32] . [Wq | Wk | Wv]   (8 k-steps)
//   logits      S = Q_h K_h^T per 8-row block of queries          (2 k-steps)
//   output      O = P_h V_h                                       (keys / 4 steps)
// The softmax runs on the S accumulators in registers: each row of an 8x8
// accumulator lives in 4 lanes, so row max and row sum take two shuffles,
// and the A operand of P V is gathered from those accumulators by shuffles.
// Rows of a centre are padded to a multiple of 8 with zero features (their
// keys are masked to -inf; their values are 0, so masked slots add exactly 0).
// Tiles of consecutive centres (padded rows <= R) stay in shared memory for
// all layers; only the final layer is written back.
#pragma once

#include "mlg_common.cuh"
#include "mlg_attn_tile.cuh"
#include "mlg_attn_hg.cuh"

namespace mlg {

__device__ __forceinline__ void dmma884(double& c0, double& c1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(c0), "+d"(c1)
               : "d"(a), "d"(b));
}

template <int R, int NT>
struct DmmaCfg {
  static constexpr int C = 32, D = 8, H = 4, N3 = 96;
  static constexpr int NB = R / 8;         // row blocks per tile (and per centre at most)
  static constexpr int XS = 36;            // strides = 4 (mod 16) doubles: conflict-free frags
  static constexpr int QS = 100;
  static constexpr int WS = 100;
  static constexpr size_t OFF_X = 0;
  static constexpr size_t OFF_Q = OFF_X + (size_t)R * XS * 8;
  static constexpr size_t OFF_W = OFF_Q + (size_t)R * QS * 8;
  static constexpr size_t OFF_S = OFF_W + (size_t)C * WS * 8;
  static constexpr size_t OFF_META = (OFF_S + (size_t)R * 8 + 15) / 16 * 16;
  static constexpr size_t SMEM = OFF_META + sizeof(TileMeta);
  static_assert(R % 8 == 0 && NT % 32 == 0, "shapes");
};

template <int R, int NT>
__global__ void __launch_bounds__(NT) k_attn_dmma(TileArgs a) {
  using Cfg = DmmaCfg<R, NT>;
  constexpr int C = Cfg::C, D = Cfg::D, H = Cfg::H, NB = Cfg::NB;
  constexpr int XS = Cfg::XS, QS = Cfg::QS, WS = Cfg::WS;
  constexpr int NW = NT / 32;
  extern __shared__ __align__(128) unsigned char smem[];
  double* sX = reinterpret_cast<double*>(smem + Cfg::OFF_X);
  double* sQ = reinterpret_cast<double*>(smem + Cfg::OFF_Q);
  double* sW = reinterpret_cast<double*>(smem + Cfg::OFF_W);
  double* sS = reinterpret_cast<double*>(smem + Cfg::OFF_S);
  TileMeta& meta = *reinterpret_cast<TileMeta*>(smem + Cfg::OFF_META);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int lr = lane >> 2, lc = lane & 3;  // fragment row / column index
  const double* G = static_cast<const double*>(a.G);
  double* out = static_cast<double*>(a.out);
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
  const double rsd = 1.0 / sqrt((double)D);

  while (true) {
    // ---- plan a tile: consecutive centres, padded rows <= R (c0[0] = first centre)
    if (tid == 0) {
      int c = meta.next_c, k = 0, rows = 0;
      const int c_end = meta.c_end;
      while (c < c_end) {
        const int n = (int)(a.row_ptr[c + 1] - a.row_ptr[c]);
        if (n > 0 && n <= R) break;
        ++c;
      }
      meta.c0[0] = c;
      while (c < c_end && k < 64) {
        const int n = (int)(a.row_ptr[c + 1] - a.row_ptr[c]);
        const int n8 = (n + 7) & ~7;
        if (n > R || rows + n8 > R) break;
        meta.off[0][k] = rows;
        rows += n8;
        ++k;
        ++c;
      }
      meta.off[0][k] = rows;
      meta.ncent[0] = k;
      meta.nrows[0] = rows;
      meta.next_c = c;
    }
    __syncthreads();
    const int ncent = meta.ncent[0], prow = meta.nrows[0], c0 = meta.c0[0];
    if (ncent == 0) break;
    // ---- load the tile's rows (16-byte async copies), zero the padding rows
    for (int ci = 0; ci < ncent; ++ci) {
      const int64_t g0 = a.row_ptr[c0 + ci];
      const int n = (int)(a.row_ptr[c0 + ci + 1] - g0);
      const int off = meta.off[0][ci], n8 = meta.off[0][ci + 1] - off;
      for (int e = tid; e < n8 * (C / 2); e += NT) {
        const int r = e / (C / 2), v = e - r * (C / 2);
        double* dst = sX + (off + r) * XS + 2 * v;
        if (r < n) cp_async16(dst, G + (g0 + r) * C + 2 * v);
        else dst[0] = dst[1] = 0.0;
      }
      for (int r = tid; r < n8; r += NT) sS[off + r] = r < n ? a.sw[g0 + r] : 0.0;
    }
    cp_async_commit();

    // weights of a layer: sW[k][m * 32 + col] = W_m[k][col]; the next layer's
    // copy starts as soon as the projection no longer reads sW
    auto load_weights = [&](int layer) {
      for (int e = tid; e < 3 * C * (C / 2); e += NT) {
        const int m = e / (C * (C / 2)), rem = e - m * C * (C / 2);
        const int k = rem / (C / 2), v = rem - k * (C / 2);
        cp_async16(sW + k * WS + m * C + 2 * v,
                   static_cast<const double*>(a.W[3 * layer + m]) + k * C + 2 * v);
      }
      cp_async_commit();
    };
    load_weights(0);
    for (int layer = 0; layer < a.n_layers; ++layer) {
      cp_async_wait<0>();
      __syncthreads();

      // ---- projection: pairs of 8x8 output blocks (row block, two adjacent
      // column blocks) over the warps; the pair shares the A fragment and
      // gives two independent accumulator chains
      const int nrb = prow / 8;
      for (int item = warp; item < nrb * 6; item += NW) {
        const int mb = item / 6, nb = (item - mb * 6) * 2;
        double c0v = 0.0, c1v = 0.0, c2v = 0.0, c3v = 0.0;
#pragma unroll
        for (int k = 0; k < C / 4; ++k) {
          const double av = sX[(mb * 8 + lr) * XS + k * 4 + lc];
          const double bv0 = sW[(k * 4 + lc) * WS + nb * 8 + lr];
          const double bv1 = sW[(k * 4 + lc) * WS + nb * 8 + 8 + lr];
          dmma884(c0v, c1v, av, bv0);
          dmma884(c2v, c3v, av, bv1);
        }
        const int r = mb * 8 + lr, col = nb * 8 + 2 * lc;
        const double s = sS[r];
        // the two blocks never straddle q / k / v (32 is a multiple of 16)
        const double f = col < C ? s * rsd : (col < 2 * C ? s : 1.0);
        sQ[r * QS + col] = c0v * f;
        sQ[r * QS + col + 1] = c1v * f;
        sQ[r * QS + col + 8] = c2v * f;
        sQ[r * QS + col + 9] = c3v * f;
      }
      __syncthreads();
      if (layer + 1 < a.n_layers) load_weights(layer + 1);

      // ---- attention: items (centre, head, query row block)
      int nitems = 0;
      for (int ci = 0; ci < ncent; ++ci) nitems += ((meta.off[0][ci + 1] - meta.off[0][ci]) / 8) * H;
      for (int item = warp; item < nitems; item += NW) {
        int ci = 0, base_item = 0;
        while (true) {
          const int cnt = ((meta.off[0][ci + 1] - meta.off[0][ci]) / 8) * H;
          if (item < base_item + cnt) break;
          base_item += cnt;
          ++ci;
        }
        const int off = meta.off[0][ci];
        const int nbk = (meta.off[0][ci + 1] - off) / 8;   // key blocks of this centre
        const int n = (int)(a.row_ptr[c0 + ci + 1] - a.row_ptr[c0 + ci]);
        const int rel = item - base_item;
        const int h = rel / nbk, ib = rel - h * nbk;
        // logits of 8 query rows against all keys of the centre
        double s[NB][2];
#pragma unroll
        for (int j = 0; j < NB; ++j) {
          s[j][0] = s[j][1] = 0.0;
          if (j < nbk) {
#pragma unroll
            for (int kk = 0; kk < D / 4; ++kk) {
              const double av = sQ[(off + ib * 8 + lr) * QS + h * D + kk * 4 + lc];
              const double bv = sQ[(off + j * 8 + lr) * QS + C + h * D + kk * 4 + lc];
              dmma884(s[j][0], s[j][1], av, bv);
            }
          }
        }
        double mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < NB; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int col = j * 8 + 2 * lc + e;
            if (j >= nbk || col >= n) s[j][e] = -INFINITY;
            mx = fmax(mx, s[j][e]);
          }
        mx = fmax(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmax(mx, __shfl_xor_sync(kFull, mx, 2));
        double sum = 0.0;
#pragma unroll
        for (int j = 0; j < NB; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const double p = j < nbk ? exp(s[j][e] - mx) : 0.0;
            s[j][e] = p;
            sum += p;
          }
        sum += __shfl_xor_sync(kFull, sum, 1);
        sum += __shfl_xor_sync(kFull, sum, 2);
        // O = P V: the A operand (row lr, key 4 kk + lc) sits in lane
        // (lr, (kk & 1) * 2 + lc / 2), element lc & 1, of accumulator kk / 2
        // two accumulator chains (even / odd key steps), summed at the end
        double o0 = 0.0, o1 = 0.0, o2 = 0.0, o3 = 0.0;
        const int src_lo = (lane & ~3) | (lc >> 1), src_hi = src_lo | 2;
#pragma unroll
        for (int j = 0; j < NB; ++j) {
          if (j < nbk) {
            const double w0 = __shfl_sync(kFull, s[j][0], src_lo);
            const double w1 = __shfl_sync(kFull, s[j][1], src_lo);
            const double x0 = __shfl_sync(kFull, s[j][0], src_hi);
            const double x1 = __shfl_sync(kFull, s[j][1], src_hi);
            const double bv0 = sQ[(off + (2 * j) * 4 + lc) * QS + 2 * C + h * D + lr];
            const double bv1 = sQ[(off + (2 * j + 1) * 4 + lc) * QS + 2 * C + h * D + lr];
            dmma884(o0, o1, (lc & 1) ? w1 : w0, bv0);
            dmma884(o2, o3, (lc & 1) ? x1 : x0, bv1);
          }
        }
        o0 += o2;
        o1 += o3;
        const double inv = 1.0 / sum;
        const int r = ib * 8 + lr;
        if (r < n) {
          double* xo = sX + (off + r) * XS + h * D + 2 * lc;
          xo[0] = o0 * inv;
          xo[1] = o1 * inv;
        }
      }
      __syncthreads();
    }
    // ---- write the tile back (16-byte stores of each centre's real rows)
    for (int ci = 0; ci < ncent; ++ci) {
      const int64_t g0 = a.row_ptr[c0 + ci];
      const int n = (int)(a.row_ptr[c0 + ci + 1] - g0);
      const int off = meta.off[0][ci];
      for (int e = tid; e < n * (C / 2); e += NT) {
        const int r = e / (C / 2), v = e - r * (C / 2);
        const double2 val = *reinterpret_cast<const double2*>(sX + (off + r) * XS + 2 * v);
        *reinterpret_cast<double2*>(out + (g0 + r) * C + 2 * v) = val;
      }
    }
    __syncthreads();
  }
}

}  // namespace mlg
