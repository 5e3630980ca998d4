// mlg_attn_dmma.cuh -- fused multi-layer block-dense attention in fp64 on the
// FP64 tensor pipe (mma.sync m16n8k16 / m16n8k8 / m8n8k4 .f64, sm_100a).
//
// The per-centre attention of the NeighborGraph issue (Proposed fix: dense
// attention per centre with masks for the ragged tail, written back to the
// edge axis), for c = 32 channels, 4 heads of d = 8, in fp64.  Every product
// is an fp64 MMA:
//   K   [rows][32] = X . Wk               m16n8k16, 16-row blocks of the tile
//   V^T [32][rows] = Wv^T . X^T           m16n8k16, 8-row blocks (stored transposed)
//   Q_h [16][8]    = X . Wq_h             m16n8k16, kept in registers
//   S   [16][8]    = Q_h . K_h^T          m16n8k8 per 8-key block
//   O   [16][8]   += P . V_h              m16n8k8 per 8-key block
// A centre's last query rows, when 8 or fewer, take the same three products
// on 8-row blocks (m8n8k4), so no MMA row is padding and no query block runs
// past its centre's rows.
// A contraction may visit its k index in any order, so each one permutes it
// to suit the fragments at hand: the projections read channel 4t + m at k
// slot t + 4m (both operands then come in contiguous 16-byte pieces); the
// logits read head dimension 2t + e at k slot t + 4e, which is the column
// layout of the Q accumulator; P V reads key 2t + e at k slot t + 4e, which
// is the column layout of the S accumulator.  So Q and P never leave
// registers and need no shuffles.
// Softmax: each lane holds two query rows (g and g + 8) of every 8-key
// block.  The row maxima are taken on the integer pipe from the doubles' high
// words, the sums by two shuffles; exponentials are in base 2 (log2 e is
// folded into the Q scale) by a table-driven method, block by block, each
// block's exponentials overlapping the previous block's P V MMA.  The FP64
// MMA and the DFMA share one pipe, so the softmax keeps its FP64 work small.
// Rows of a centre are padded to a multiple of 8 with zero features (their
// keys are masked to -inf and their values are 0).
// One CTA per SM holds a tile of consecutive centres for all layers: the
// layer's input X and its output ping-pong between two buffers, and only the
// last layer's output goes back to global memory.  A layer is phase A (K and
// V^T of the whole tile) and phase B (units of equal work: one 16-row query
// block and head, or two heads of an 8-row block), with a barrier after each.
#pragma once

#include "mlg_common.cuh"
#include "mlg_attn_tile.cuh"
#include "mlg_attn_hg.cuh"

namespace mlg {

// C[8x8] += A[8x4] B[4x8] (fp64): lane (g, t) holds A(g, t), B(t, g) and
// C(g, 2t), C(g, 2t + 1).
__device__ __forceinline__ void dmma884(double& c0, double& c1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(c0), "+d"(c1)
               : "d"(a), "d"(b));
}

// Query blocks of a centre with n edges: 16-row blocks (the last one may
// be partial when more than 8 rows remain) and at most one final 8-row block.
__host__ __device__ __forceinline__ int full_qblocks(int n) {
  return n / 16 + (n % 16 > 8 ? 1 : 0);
}
__host__ __device__ __forceinline__ int half_qblocks(int n) {
  return n % 16 != 0 && n % 16 <= 8 ? 1 : 0;
}

// C[16x8] += A[16x8] B[8x8] (fp64).  Lane (g, t) = (lane / 4, lane % 4) holds
// a = {A(g,t), A(g+8,t), A(g,t+4), A(g+8,t+4)}, b = {B(t,g), B(t+4,g)},
// c = {C(g,2t), C(g,2t+1), C(g+8,2t), C(g+8,2t+1)}.
__device__ __forceinline__ void dmma_k8(double (&c)[4], double a0, double a1, double a2, double a3,
                                        double b0, double b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f64.f64.f64.f64 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+d"(c[0]), "+d"(c[1]), "+d"(c[2]), "+d"(c[3])
      : "d"(a0), "d"(a1), "d"(a2), "d"(a3), "d"(b0), "d"(b1));
}

// C[16x8] += A[16x16] B[16x8] (fp64): a[i] = A(g + 8 (i % 2), t + 4 (i / 2)),
// b[i] = B(t + 4 i, g), c as in dmma_k8.
__device__ __forceinline__ void dmma_k16(double (&c)[4], const double (&a)[8],
                                         const double (&b)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f64.f64.f64.f64 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7,%8,%9,%10,%11}, {%12,%13,%14,%15}, {%0,%1,%2,%3};"
      : "+d"(c[0]), "+d"(c[1]), "+d"(c[2]), "+d"(c[3])
      : "d"(a[0]), "d"(a[1]), "d"(a[2]), "d"(a[3]), "d"(a[4]), "d"(a[5]), "d"(a[6]), "d"(a[7]),
        "d"(b[0]), "d"(b[1]), "d"(b[2]), "d"(b[3]));
}

// 2^y for y <= 0, or slightly above (-inf -> 0, NaN -> NaN, +inf -> +inf), after P. T. P.
// Tang's table-driven exponential (ACM TOMS 15(2), 1989), in base 2:
// k = rint(1024 y), r = y - k / 1024 (exact, |r| <= 1/2048),
// 2^y = 2^(k >> 10) 2^((k & 1023) / 1024) 2^r, with the 1024 values
// 2^(j/1024) in a shared-memory table `tab` and 2^r = exp(r ln 2) by its
// Taylor series to degree 3 (truncation below 5.6e-16 relative, as
// |r ln 2| <= 3.4e-4).  Arguments whose high word lies below that of -1000
// give 0 (the true value is below 1e-301); above that the scaling by
// 2^(k >> 10) is an add to the exponent field that stays in the normal range.
// Besides the table load, the only FP64-pipe work is six operations.
namespace exp2tab {
constexpr int kBits = 10, kSize = 1 << kBits;
constexpr double kLn2 = 0.693147180559945309417232121458176568;
constexpr double c1 = kLn2, c2 = c1 * kLn2 / 2, c3 = c2 * kLn2 / 3;
constexpr double kRound = 6755399441055744.0;  // 1.5 * 2^52: adding it rounds to an integer
constexpr unsigned kHiMinus1000 = 0xC08F4000u;  // high word of -1000.0
}  // namespace exp2tab

// fills tab[0 .. 1023] with 2^(j/1024), threads tid0, tid0 + stride, ...
__device__ __forceinline__ void exp2_table_fill(double* tab, int tid0, int stride) {
  for (int j = tid0; j < exp2tab::kSize; j += stride) tab[j] = exp2((double)j / exp2tab::kSize);
}

__device__ __forceinline__ double exp2_neg(double y, const double* tab) {
  double kd = fma(y, (double)exp2tab::kSize, exp2tab::kRound);
  const int k = __double2loint(kd);
  kd -= exp2tab::kRound;
  const double r = fma(kd, -1.0 / exp2tab::kSize, y);
  double p = exp2tab::c3;
  p = fma(p, r, exp2tab::c2);
  p = fma(p, r, exp2tab::c1);
  p = fma(p, r, 1.0);
  const double v = tab[k & (exp2tab::kSize - 1)] * p;
  const double out =
      __hiloint2double(__double2hiint(v) + ((k >> exp2tab::kBits) << 20), __double2loint(v));
  const unsigned hy = (unsigned)__double2hiint(y);
  double res = hy > exp2tab::kHiMinus1000 ? 0.0 : out;  // below -1000, and -inf: 0
  if ((hy & 0x7ff00000u) == 0x7ff00000u && (hy != 0xfff00000u || __double2loint(y) != 0))
    res = y;  // NaN and +inf give themselves
  return res;
}

// Order-preserving integer image of a double's high word (sign folded), for
// row maxima on the integer pipe; from_ord_hi inverts it with a zero low
// word, which is within 2^-20 relative of the maximum: the softmax does not
// depend on the shift, and the exponential takes arguments slightly above 0.
__device__ __forceinline__ int ord_hi(double x) {
  const int h = __double2hiint(x);
  return h ^ ((h >> 31) & 0x7fffffff);
}
__device__ __forceinline__ double from_ord_hi(int o) {
  return __hiloint2double(o ^ ((o >> 31) & 0x7fffffff), 0);
}

// out[i] = exp2_neg(y[i]) (diagnostics).
__global__ void k_exp2_neg(const double* y, double* out, int64_t n) {
  __shared__ double tab[exp2tab::kSize];
  exp2_table_fill(tab, threadIdx.x, blockDim.x);
  __syncthreads();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = exp2_neg(y[i], tab);
}

__device__ __forceinline__ double2 lds2(const double* p) {
  return *reinterpret_cast<const double2*>(p);
}
__device__ __forceinline__ void sts2(double* p, double x, double y) {
  *reinterpret_cast<double2*>(p) = make_double2(x, y);
}

// Fragment A of a 16-row m16n8k16 block from a row-major [rows][stride]
// array at `p` = row g, column 4 t (+ k0): channels 4t .. 4t + 3 of rows g and
// g + 8 in k slots t, t + 4, t + 8, t + 12.
__device__ __forceinline__ void frag_a16(double (&av)[8], const double* p, int stride) {
  double2 v;
  v = lds2(p);              av[0] = v.x; av[2] = v.y;
  v = lds2(p + 2);          av[4] = v.x; av[6] = v.y;
  v = lds2(p + 8 * stride); av[1] = v.x; av[3] = v.y;
  v = lds2(p + 8 * stride + 2); av[5] = v.x; av[7] = v.y;
}
// Fragment B (k slots t + 4i, i = 0..3) from the same channel-contiguous
// layout, column g of the product = row g of the array.
__device__ __forceinline__ void frag_b16(double (&bv)[4], const double* p) {
  double2 v;
  v = lds2(p);     bv[0] = v.x; bv[1] = v.y;
  v = lds2(p + 2); bv[2] = v.x; bv[3] = v.y;
}
// Fragment B from a [k][stride] weight array at `p` = row 4t (+ k0), column
// g of the product: rows 4t .. 4t + 3 in k slots t + 4i.
__device__ __forceinline__ void frag_bw(double (&bv)[4], const double* p, int stride) {
#pragma unroll
  for (int i = 0; i < 4; ++i) bv[i] = p[i * stride];
}
// Fragment A of the transposed weights (rows of the product = columns g,
// g + 8 of the array) from a [k][stride] array at `p` = row 4t (+ k0),
// column g.
__device__ __forceinline__ void frag_aw(double (&av)[8], const double* p, int stride) {
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    av[2 * m] = p[m * stride];
    av[2 * m + 1] = p[m * stride + 8];
  }
}

// R: tile rows (centres padded to 8 rows, packed); NBC: key blocks of 8 per
// centre at most (centres with more than 8 NBC edges are not taken).
template <int R, int NBC, int NT>
struct DmmaCfg {
  static constexpr int C = 32, D = 8, H = 4;
  static constexpr int RA = R + 8;   // + slack read by 16-row blocks past the last centre
  static constexpr int XS = 34;      // row strides in doubles, chosen so that the
  static constexpr int KS = 40;      // 16-byte fragment loads and stores of every
  static constexpr int VS = RA;      // phase are free of bank conflicts
  static constexpr int WS = 3 * C + 1;  // W rows: odd, so 8-byte fragment loads of rows 4t + i
                                        // fill a half-warp's banks once
  static constexpr size_t XBYTES = (size_t)RA * XS * 8;
  static constexpr size_t OFF_X = 0;                               // [2][RA][XS]
  static constexpr size_t OFF_K = OFF_X + 2 * XBYTES;              // [RA][KS]
  static constexpr size_t OFF_V = OFF_K + (size_t)RA * KS * 8;     // [C][VS]  (V^T)
  static constexpr size_t OFF_W = OFF_V + (size_t)C * VS * 8;      // [C][WS]: [Wq | Wk | Wv]
  static constexpr size_t OFF_S = OFF_W + (size_t)C * WS * 8;      // [RA]
  static constexpr size_t OFF_T = (OFF_S + (size_t)RA * 8 + 15) / 16 * 16;  // exp2 table
  static constexpr size_t OFF_META = OFF_T + (size_t)exp2tab::kSize * 8;
  static constexpr size_t SMEM = OFF_META + sizeof(TileMeta);
  static_assert(R % 16 == 0 && VS % 16 == 8 && NBC * 8 <= R && NT % 32 == 0, "shapes");
};

template <int R, int NBC, int NT>
__global__ void __launch_bounds__(NT, 1) k_attn_dmma(TileArgs a) {
  using Cfg = DmmaCfg<R, NBC, NT>;
  constexpr int C = Cfg::C, D = Cfg::D, H = Cfg::H, RA = Cfg::RA;
  constexpr int XS = Cfg::XS, KS = Cfg::KS, VS = Cfg::VS, WS = Cfg::WS;
  constexpr int NW = NT / 32;
  extern __shared__ __align__(128) unsigned char smem[];
  double* sXb = reinterpret_cast<double*>(smem + Cfg::OFF_X);
  double* sK = reinterpret_cast<double*>(smem + Cfg::OFF_K);
  double* sV = reinterpret_cast<double*>(smem + Cfg::OFF_V);
  double* sW = reinterpret_cast<double*>(smem + Cfg::OFF_W);
  double* sS = reinterpret_cast<double*>(smem + Cfg::OFF_S);
  double* tab = reinterpret_cast<double*>(smem + Cfg::OFF_T);
  TileMeta& meta = *reinterpret_cast<TileMeta*>(smem + Cfg::OFF_META);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
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
  exp2_table_fill(tab, tid, NT);
  const double qscale = 1.4426950408889634 / sqrt((double)D);  // log2(e) / sqrt(d)
  __syncthreads();

  // weights: sW[k][m C + col] = W_m[k][col] (m = 0, 1, 2: q, k, v), copied
  // by 8-byte async copies (the row stride is odd); a layer's q block and its
  // k, v blocks are copied at different times (see the layer loop)
  auto load_w = [&](int layer, int m0, int nm) {
    for (int e = tid; e < nm * C * C; e += NT) {
      const int m = m0 + e / (C * C), rem = e % (C * C);
      const int k = rem / C, col = rem % C;
      cp_async8(sW + k * WS + m * C + col,
                static_cast<const double*>(a.W[3 * layer + m]) + k * C + col);
    }
    cp_async_commit();
  };

  // Attention of query rows qb * 16 .. + 15 of the centre at tile row `off`
  // (n edges, nkb key blocks), head h: X from sX, output rows to sXn.
  auto attend16 = [&](const double* sX, double* sXn, int off, int n, int nkb, int qb, int h) {
    const int q0 = off + qb * 16;          // first query row of the block (tile-local)
    const bool hi_rows = qb * 16 + 8 < n;  // rows g + 8 hold queries
    // Q_h of the block: q[e] = Q(g, 2t + e), q[2 + e] = Q(g + 8, 2t + e)
    double q[4] = {0.0, 0.0, 0.0, 0.0};
    {
      const double* xr = sX + (q0 + g) * XS + 4 * t;
      const double* wr = sW + 4 * t * WS + h * D + g;
#pragma unroll
      for (int k0 = 0; k0 < C; k0 += 16) {
        double av[8], bv[4];
        frag_a16(av, xr + k0, XS);
        frag_bw(bv, wr + k0 * WS, WS);
        dmma_k16(q, av, bv);
      }
      const double f0 = sS[q0 + g] * qscale, f1 = sS[q0 + g + 8] * qscale;
      q[0] *= f0;
      q[1] *= f0;
      q[2] *= f1;
      q[3] *= f1;
    }
    // logits against the centre's keys (base-2 units):
    // s[j][e] = S(g, 8j + 2t + e), s[j][2 + e] = S(g + 8, 8j + 2t + e)
    double s[NBC][4];
#pragma unroll
    for (int j = 0; j < NBC; ++j) {
      s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.0;
      if (j < nkb) {
        const double2 kv = lds2(sK + (off + 8 * j + g) * KS + h * D + 2 * t);
        dmma_k8(s[j], q[0], q[2], q[1], q[3], kv.x, kv.y);
      }
    }
    int o0 = INT_MIN, o1 = INT_MIN;  // row maxima, on the integer pipe
#pragma unroll
    for (int j = 0; j < NBC; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool valid = j < nkb && 8 * j + 2 * t + e < n;
        s[j][e] = valid ? s[j][e] : -INFINITY;
        s[j][2 + e] = valid ? s[j][2 + e] : -INFINITY;
        o0 = max(o0, ord_hi(s[j][e]));
        o1 = max(o1, ord_hi(s[j][2 + e]));
      }
    o0 = max(o0, __shfl_xor_sync(kFull, o0, 1));
    o0 = max(o0, __shfl_xor_sync(kFull, o0, 2));
    o1 = max(o1, __shfl_xor_sync(kFull, o1, 1));
    o1 = max(o1, __shfl_xor_sync(kFull, o1, 2));
    const double m0 = from_ord_hi(o0), m1 = from_ord_hi(o1);
    // weights and O = P V_h block by block (a block's exponentials overlap
    // the previous block's MMA), two accumulator chains (even / odd blocks)
    double l0 = 0.0, l1 = 0.0;
    double o[2][4] = {{0.0, 0.0, 0.0, 0.0}, {0.0, 0.0, 0.0, 0.0}};
#pragma unroll
    for (int j = 0; j < NBC; ++j) {
      if (j < nkb) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          s[j][e] = exp2_neg(s[j][e] - m0, tab);
          l0 += s[j][e];
          if (hi_rows) {
            s[j][2 + e] = exp2_neg(s[j][2 + e] - m1, tab);
            l1 += s[j][2 + e];
          } else {
            s[j][2 + e] = 0.0;
          }
        }
        const double2 vv = lds2(sV + (h * D + g) * VS + off + 8 * j + 2 * t);
        dmma_k8(o[j & 1], s[j][0], s[j][2], s[j][1], s[j][3], vv.x, vv.y);
      }
    }
    l0 += __shfl_xor_sync(kFull, l0, 1);
    l0 += __shfl_xor_sync(kFull, l0, 2);
    l1 += __shfl_xor_sync(kFull, l1, 1);
    l1 += __shfl_xor_sync(kFull, l1, 2);
    const int r = qb * 16 + g;
    if (r < n) {
      const double i0 = 1.0 / l0;
      sts2(sXn + (q0 + g) * XS + h * D + 2 * t, (o[0][0] + o[1][0]) * i0,
           (o[0][1] + o[1][1]) * i0);
    }
    if (r + 8 < n) {
      const double i1 = 1.0 / l1;
      sts2(sXn + (q0 + g + 8) * XS + h * D + 2 * t, (o[0][2] + o[1][2]) * i1,
           (o[0][3] + o[1][3]) * i1);
    }
  };
  // The same for the 8 query rows qr .. qr + 7 of the centre (m8n8k4): the
  // projection's step s reads channel 16 (s / 4) + 4t + s % 4 at k slot t, the
  // logits and P V read dimension / key 2t + e at the k slot t of step e.
  auto attend8 = [&](const double* sX, double* sXn, int off, int n, int nkb, int qr, int h) {
    const int q0 = off + qr;
    double qa[2] = {0.0, 0.0}, qb[2] = {0.0, 0.0};  // two chains: channels 0..15, 16..31
    {
      const double* xr = sX + (q0 + g) * XS + 4 * t;
      const double* wr = sW + 4 * t * WS + h * D + g;
#pragma unroll
      for (int c16 = 0; c16 < C; c16 += 16) {
        double* q = c16 ? qb : qa;
        const double2 xa = lds2(xr + c16), xb = lds2(xr + c16 + 2);
        dmma884(q[0], q[1], xa.x, wr[(c16 + 0) * WS]);
        dmma884(q[0], q[1], xa.y, wr[(c16 + 1) * WS]);
        dmma884(q[0], q[1], xb.x, wr[(c16 + 2) * WS]);
        dmma884(q[0], q[1], xb.y, wr[(c16 + 3) * WS]);
      }
    }
    const double f = sS[q0 + g] * qscale;
    const double q0v = (qa[0] + qb[0]) * f, q1v = (qa[1] + qb[1]) * f;  // Q(g, 2t), Q(g, 2t + 1)
    // s[j][e] = S(g, 8j + 2t + e)
    double s[NBC][2];
#pragma unroll
    for (int j = 0; j < NBC; ++j) {
      s[j][0] = s[j][1] = 0.0;
      if (j < nkb) {
        const double2 kv = lds2(sK + (off + 8 * j + g) * KS + h * D + 2 * t);
        dmma884(s[j][0], s[j][1], q0v, kv.x);
        dmma884(s[j][0], s[j][1], q1v, kv.y);
      }
    }
    int om = INT_MIN;
#pragma unroll
    for (int j = 0; j < NBC; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool valid = j < nkb && 8 * j + 2 * t + e < n;
        s[j][e] = valid ? s[j][e] : -INFINITY;
        om = max(om, ord_hi(s[j][e]));
      }
    om = max(om, __shfl_xor_sync(kFull, om, 1));
    om = max(om, __shfl_xor_sync(kFull, om, 2));
    const double m = from_ord_hi(om);
    double l = 0.0;
    double o[2][2] = {{0.0, 0.0}, {0.0, 0.0}};
#pragma unroll
    for (int j = 0; j < NBC; ++j) {
      if (j < nkb) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          s[j][e] = exp2_neg(s[j][e] - m, tab);
          l += s[j][e];
        }
        const double2 vv = lds2(sV + (h * D + g) * VS + off + 8 * j + 2 * t);
        dmma884(o[j & 1][0], o[j & 1][1], s[j][0], vv.x);
        dmma884(o[j & 1][0], o[j & 1][1], s[j][1], vv.y);
      }
    }
    l += __shfl_xor_sync(kFull, l, 1);
    l += __shfl_xor_sync(kFull, l, 2);
    if (qr + g < n) {
      const double il = 1.0 / l;
      sts2(sXn + (q0 + g) * XS + h * D + 2 * t, (o[0][0] + o[1][0]) * il,
           (o[0][1] + o[1][1]) * il);
    }
  };

  while (true) {
    // ---- plan a tile: consecutive centres with 1 .. 8 NBC edges, each padded
    // to a multiple of 8 rows, padded rows <= R
    if (tid == 0) {
      int c = meta.next_c, k = 0, rows = 0, tasks = 0;
      const int c_end = meta.c_end;
      while (c < c_end) {
        const int n = (int)(a.row_ptr[c + 1] - a.row_ptr[c]);
        if (n > 0 && n <= NBC * 8 && n <= a.nnei_max) break;
        if (n > a.nnei_max) atomicOr(a.status, (uint32_t)MLG_STATUS_ROW_TOO_LONG);
        ++c;
      }
      meta.c0[0] = c;
      while (c < c_end && k < 64) {
        const int n = (int)(a.row_ptr[c + 1] - a.row_ptr[c]);
        const int n8 = (n + 7) & ~7;
        if (n > NBC * 8 || n > a.nnei_max || rows + n8 > R) break;
        meta.off[0][k] = rows;
        meta.task0[0][k] = tasks;
        tasks += H * full_qblocks(n) + (H / 2) * half_qblocks(n);
        rows += n8;
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
    const int ncent = meta.ncent[0], prow = meta.nrows[0], c0 = meta.c0[0];
    const int ntask = meta.task0[0][ncent];
    if (ncent == 0) break;

    // ---- load the tile: each centre's rows by 16-byte async copies into
    // buffer 0; padding rows and the slack zero in both buffers
    for (int ci = 0; ci < ncent; ++ci) {
      const int64_t g0 = a.row_ptr[c0 + ci];
      const int n = (int)(a.row_ptr[c0 + ci + 1] - g0);
      const int off = meta.off[0][ci], n8 = meta.off[0][ci + 1] - off;
      for (int e = tid; e < n * (C / 2); e += NT) {
        const int r = e / (C / 2), v = e - r * (C / 2);
        cp_async16(sXb + (off + r) * XS + 2 * v, G + (g0 + r) * C + 2 * v);
      }
      for (int e = tid; e < (n8 - n) * (C / 2); e += NT) {
        const int r = off + n + e / (C / 2), v = e % (C / 2);
        sts2(sXb + r * XS + 2 * v, 0.0, 0.0);
        sts2(sXb + (RA + r) * XS + 2 * v, 0.0, 0.0);
      }
      for (int r = tid; r < n8; r += NT) sS[off + r] = r < n ? a.sw[g0 + r] : 0.0;
    }
    cp_async_commit();
    for (int e = tid; e < (RA - prow) * (C / 2); e += NT) {
      const int r = prow + e / (C / 2), v = e % (C / 2);
      sts2(sXb + r * XS + 2 * v, 0.0, 0.0);
      sts2(sXb + (RA + r) * XS + 2 * v, 0.0, 0.0);
    }
    for (int r = prow + tid; r < RA; r += NT) sS[r] = 0.0;
    load_w(0, 0, 3);
    cp_async_wait<0>();
    __syncthreads();

    const int nrb16 = (prow + 15) / 16;  // 16-row blocks of the tile
    for (int layer = 0; layer < a.n_layers; ++layer) {
      const double* sX = sXb + (layer & 1) * RA * XS;
      double* sXn = sXb + ((layer + 1) & 1) * RA * XS;
      // this layer's Wq is copied during phase A (the previous layer's
      // phase B was its last reader)
      if (layer > 0) load_w(layer, 0, 1);

      // ---- phase A: K (16-row blocks x pairs of 8-column blocks) and V^T
      // (16-dimension blocks x pairs of 8-row blocks); 4 MMAs per item
      const int nka = nrb16 * 2;
      for (int item = warp; item < 2 * nka; item += NW) {
        double c[2][4] = {{0.0, 0.0, 0.0, 0.0}, {0.0, 0.0, 0.0, 0.0}};
        if (item < nka) {
          const int rb = item >> 1, cb = (item & 1) * 2;  // rows 16 rb.., columns 8 cb .. 8 cb + 15
          const double* xr = sX + (rb * 16 + g) * XS + 4 * t;
          const double* wr = sW + 4 * t * WS + C + cb * 8 + g;
#pragma unroll
          for (int k0 = 0; k0 < C; k0 += 16) {
            double av[8], b0[4], b1[4];
            frag_a16(av, xr + k0, XS);
            frag_bw(b0, wr + k0 * WS, WS);
            frag_bw(b1, wr + k0 * WS + 8, WS);
            dmma_k16(c[0], av, b0);
            dmma_k16(c[1], av, b1);
          }
          const int r = rb * 16 + g;
          const double s0 = sS[r], s1 = sS[r + 8];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            double* kr = sK + r * KS + (cb + j) * 8 + 2 * t;
            sts2(kr, c[j][0] * s0, c[j][1] * s0);
            sts2(kr + 8 * KS, c[j][2] * s1, c[j][3] * s1);
          }
        } else {
          const int it = item - nka;
          const int db = it & 1, rb = it >> 1;  // dimensions 16 db.., rows 16 rb..
          const double* wr = sW + 4 * t * WS + 2 * C + db * 16 + g;
          const double* xr = sX + (rb * 16 + g) * XS + 4 * t;
#pragma unroll
          for (int k0 = 0; k0 < C; k0 += 16) {
            double av[8], b0[4], b1[4];
            frag_aw(av, wr + k0 * WS, WS);
            frag_b16(b0, xr + k0);
            frag_b16(b1, xr + 8 * XS + k0);
            dmma_k16(c[0], av, b0);
            dmma_k16(c[1], av, b1);
          }
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            double* vr = sV + (db * 16 + g) * VS + rb * 16 + j * 8 + 2 * t;
            sts2(vr, c[j][0], c[j][1]);
            sts2(vr + 8 * VS, c[j][2], c[j][3]);
          }
        }
      }
      cp_async_wait<0>();
      __syncthreads();

      // the next layer's Wk, Wv are copied during phase B (phase A above was
      // their last reader)
      if (layer + 1 < a.n_layers) load_w(layer + 1, 1, 2);

      // ---- phase B: units of equal work: (centre, 16-row query block, head),
      // or two heads of a centre's final 8-row query block
      for (int unit = warp; unit < ntask; unit += NW) {
        int ci = 0;
        while (meta.task0[0][ci + 1] <= unit) ++ci;
        const int off = meta.off[0][ci];
        const int n = (int)(a.row_ptr[c0 + ci + 1] - a.row_ptr[c0 + ci]);
        const int nkb = (meta.off[0][ci + 1] - off) >> 3;
        const int nf = full_qblocks(n);
        const int rel = unit - meta.task0[0][ci];
        if (rel < H * nf) {
          attend16(sX, sXn, off, n, nkb, rel / H, rel % H);
        } else {
          const int h0 = 2 * (rel - H * nf);
          attend8(sX, sXn, off, n, nkb, nf * 16, h0);
          attend8(sX, sXn, off, n, nkb, nf * 16, h0 + 1);
        }
      }
      cp_async_wait<0>();
      __syncthreads();
    }
    // ---- write the tile back (16-byte stores of each centre's real rows)
    const double* sR = sXb + (a.n_layers & 1) * RA * XS;
    for (int ci = 0; ci < ncent; ++ci) {
      const int64_t g0 = a.row_ptr[c0 + ci];
      const int n = (int)(a.row_ptr[c0 + ci + 1] - g0);
      const int off = meta.off[0][ci];
      for (int e = tid; e < n * (C / 2); e += NT) {
        const int r = e / (C / 2), v = e - r * (C / 2);
        *reinterpret_cast<double2*>(out + (g0 + r) * C + 2 * v) =
            lds2(sR + (off + r) * XS + 2 * v);
      }
    }
    __syncthreads();
  }
}

}  // namespace mlg
