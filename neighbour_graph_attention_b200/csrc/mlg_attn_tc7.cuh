// mlg_attn_tc7.cuh -- fp32 block-dense attention, 32 channels, 4 heads of 8,
// one layer, centres of 1..64 edges: the projection and the logits on the
// 5th-generation tensor cores (tcgen05.mma kind::tf32, 3xTF32), the softmax
// on the SIMT units and the weighted sum P V on warp-level tensor-core MMAs
// (mma.sync m16n8k16, fp16 operands split hi + lo, fp32 accumulation), one
// group of four warps per head that also reads back its own head's q, k, v.
//
// Per centre i with n edges (NeighborGraph issue, Proposed fix: each
// centre's edges are one small dense block, attended to with dense
// products, unequal lengths masked per row, outputs returned to the edges):
//   q_a = s_a G_a Wq log2(e)/sqrt(d),  k_b = s_b G_b Wk,  v_b = G_b Wv
//   S_ab = q_a . k_b (per head),  P_ab = 2^(S_ab - max_b S_ab),
//   O_a = sum_b P_ab v_b / sum_b P_ab.
//
// Division of the work: a tcgen05.mma of M = 128 and K = 8 takes a fixed
// ~49 cycles up to N = 64, so the contraction over a centre's keys (P V,
// N = d = 8 per head) does not pay on tcgen05; from registers on the FP32
// pipe it is bound by the shared-memory loads of v (each broadcast 16-byte
// load costs two cycles and feeds one row).  The logits contract over d = 8:
// one tcgen05 instruction per term, head and centre.  P V runs on warp-level
// MMAs: the logits are read from TMEM with the 16x256b shape, which hands
// each thread the accumulator-fragment positions of an m16n8 tile (rows g and
// g + 8, columns 2c and 2c + 1 of every 8), the very positions of the A
// fragment of m16n8k16, so P never moves between threads.
//
// Tiles of 128 rows hold up to two centres, each starting at a multiple of
// 32 rows, so that every warp's TMEM lane quadrant belongs to one centre.
//   projection  D[128 x 96] = X[128 x 32] . [Wq|Wk|Wv], 3xTF32 (12 MMAs):
//               A hi is the slab as TMA landed it (the tensor core reads the
//               leading 19 bits of each fp32 value), A lo = x - those bits
//               (formed by the groups, two float4 per thread)
//   read-back   group h reads its head's q (scaled by s_a log2(e)/sqrt(d))
//               and k (scaled by s_b) back and splits them into TF32 hi / lo
//               operands: q into TMEM, the A operand of its row's centre
//               (the other centre's operand gets a zero row), k into its
//               centre's K-major shared-memory key operand at the key's
//               slot; v as fp32 rows with the two keys of a pair
//               interleaved (two buffers per head, alternating between tiles)
//   logits      per head, in the order the groups finish reading back: for each
//               centre c, S[128 x N] += Q_h^c . (K_h^c)^T, 3 MMAs (lo.hi,
//               hi.lo, hi.hi) with N the tile's longest row in 16s.  The zero
//               rows make each centre's MMAs add exactly 0 to the other
//               centre's rows, so one buffer of N <= 64 columns holds every
//               row's logits over its own keys: each head has a buffer of
//               its own (64 columns), and a group never waits for another.
//               k is kept finite (a NaN or infinite k becomes 0) so that a
//               zero row times it stays 0; the centre still turns NaN
//               through its v.
//   group h     head h, per block of 16 rows: S from TMEM (16x256b), the row
//               maxima over the four threads of a quad, 2^(S - max) on the
//               special-function unit, the sums, then per 16 keys
//               O += P_hi V_hi + P_hi V_lo + P_lo V_hi (three m16n8k16 MMAs):
//               P = P_hi + P_lo with P_hi = P rounded to a multiple of 2^-11
//               and both halves fp16; v scaled by a power of two (the tile's
//               largest |v| of the head into [2^13, 2^14): no fp16 value
//               overflows, and the lo halves of small v stay normal) and
//               split the same way.  The rounding left is about 2^-22 of
//               each product plus 2^-24 absolute on the weights, far inside
//               fp32 tolerance (a numpy model of these splits is among the
//               tests).
//   output      O 2^e / sum straight to global memory: each quad writes one
//               whole 32-byte sector of an output row
// A group's next read-back comes after its softmax, so its logits buffer is
// free by then: the only waits between a group and the tensor pipe are the
// projection of the next tile (issued early) and its own logits.
//
// Warp roles (576 threads, one CTA per SM):
//   warp 0      issues every MMA (one elected thread)
//   warp 1      plans tiles two ahead (a window of row starts in the lanes)
//               and loads each slab with 2-D TMA boxes of {4 channels x 32
//               rows}, one per lane, straight into the K-major operand
//               layout (two slab slots)
//   warps 2-17  four groups of four warps, group h: the read-back of head h,
//               a share of the next tile's A lo, the softmax and P V of head h
// Every wait is bounded; on expiry the kernel records MLG_STATUS_TIMEOUT,
// every role leaves its loop, the MMA thread waits for its own MMAs and the
// producer for the slab copies in flight before TMEM is freed.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "mlg_common.cuh"
#include "mlg_attn_tile.cuh"
#include "mlg_attn_tc.cuh"
#include "mlg_attn_tc2.cuh"

namespace mlg {

namespace tc7 {

using tc2::Plan;
using tc2::Waiter;
using tc2::centre_of_group;
using tc2::ex2;
using tc2::idesc_tf32;
using tc2::mbar_arrive;
using tc2::tmem_st16;
using tc2::tmem_wait_st;
using tc2::umma_tf32_ts;

constexpr int C = 32, D = 8, H = 4, N3 = 96, R = 128;
constexpr int MAXN = 64;        // most edges of a centre handled here
constexpr int NG = 4;           // compute groups (one per head)
constexpr int GT = 128;         // threads per compute group
constexpr int NT = 64 + NG * GT;
constexpr int VS2 = 2 * C + 4;  // floats per key pair of V: [head][t][2 keys], padded

// TMEM columns (512 allocated)
constexpr uint32_t T_PROJ = 0;    // projection D: q 0-31, k 32-63, v 64-95
constexpr uint32_t T_S = 128;     // logits of head h: T_S + 64 h, [128 rows x 64 keys]
constexpr uint32_t T_Q = 384;     // q operands of head h: T_Q + 32 h + 16 c + 8 m
                                  // (centre c, m 0 hi / 1 lo), [128 rows x 8]

// shared memory layout (bytes)
constexpr size_t W_BYTES = (size_t)N3 * C * 4;          // one of W hi / lo (B operand)
constexpr size_t A_BYTES = (size_t)R * C * 4;           // one of X hi / lo, the raw slab
constexpr size_t K_BYTES = (size_t)MAXN * D * 4;        // one (head, centre) k operand, hi or lo
constexpr size_t V_BYTES = (size_t)(R / 2) * VS2 * 4;   // one V buffer
constexpr size_t OFF_WHI = 0;
constexpr size_t OFF_WLO = OFF_WHI + W_BYTES;
constexpr size_t OFF_X = OFF_WLO + W_BYTES;             // 2 slabs (TMA targets, A hi)
constexpr size_t OFF_ALO = OFF_X + 2 * A_BYTES;         // A lo of the next projection
constexpr size_t OFF_K = OFF_ALO + A_BYTES;             // [head][centre][hi, lo]
constexpr size_t OFF_V = OFF_K + 4 * H * K_BYTES;       // 2 x [64 key pairs][VS2] fp32
constexpr size_t OFF_META = OFF_V + 2 * V_BYTES;

// operand of (head h, centre c, part m: 0 hi, 1 lo)
__host__ __device__ constexpr size_t k_off(int h, int c, int m) {
  return OFF_K + (size_t)((h * 2 + c) * 2 + m) * K_BYTES;
}

struct Meta {
  Plan plan[4];             // ring of four: tile t in slot t % 4
  int fail;
  uint32_t tmem;
  int nissued[2];           // slab copies issued into each slot
  uint64_t bar_xfull[2];    // slab and plan of ring slot landed (TMA tx)
  uint64_t bar_w;           // weights split, key operands zeroed (count NG * GT)
  uint64_t bar_a;           // A lo of a tile written, or no tile left (count NG * GT)
  uint64_t bar_proj;        // projection done (commit)
  uint64_t bar_qk[H];       // q and k of head h in shared memory (count GT)
  uint64_t bar_s[H];        // logits of head h done (commit)
  uint64_t bar_vg[H];       // group h has written its v rows of a tile (count GT)
  uint64_t bar_fin;         // every MMA of the CTA done (commit, at exit)
  uint32_t vmax[H][2][4];   // per head, tile parity and warp: bits of the largest finite |v|
};
constexpr size_t SMEM = OFF_META + sizeof(Meta);
static_assert(SMEM <= 227 * 1024, "shared memory");
static_assert(SMEM > 116 * 1024, "one CTA per SM (the kernel holds all 512 TMEM columns)");

// What a compute thread needs of a tile: its warp's centre, that centre's
// edges and first tile row, and its own row's place in the output.
struct RowInfo {
  int ncent;       // centres in the tile (0: no work left)
  int cw;          // the warp's centre (-1: none)
  int nrow;        // its edges
  int key0;        // its first tile row
  long long orow;  // edge index of this thread's row (valid when vrow)
  long long obase; // edge index of tile row r of the centre: obase + r
  bool vrow;       // the row is one of the centre's edges
  double sw;       // s of that edge (0 otherwise)
};

// 16 TMEM lanes x 64 columns in the 16x256b shape (x8): thread t gets, for
// each 8-column chunk k, v[4k..4k+3] = (lane g, column 8k+2c), (g, 8k+2c+1),
// (g+8, 8k+2c), (g+8, 8k+2c+1), with g = t / 4 and c = t % 4 (the m16n8
// accumulator-fragment positions).
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t addr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
        "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
        "=r"(v[31])
      : "r"(addr));
}

// D += A B, m16n8k16, fp16 operands, fp32 accumulators
__device__ __forceinline__ void mma_f16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// (p0, p1) in [0, 1] -> fp16x2 hi and lo, p = hi + lo: hi is p rounded to a
// multiple of 2^-11 by adding and removing 2^12 (exact in fp16), lo the rest
// (|lo| <= 2^-12, rounded to fp16: at most 2^-24 off)
__device__ __forceinline__ void split_p_f16x2(float p0, float p1, uint32_t& hi, uint32_t& lo) {
  const float2 c = make_float2(4096.f, 4096.f), nc = make_float2(-4096.f, -4096.f);
  const float2 p = make_float2(p0, p1);
  const float2 h = __fadd2_rn(__fadd2_rn(p, c), nc);
  const float2 l = __fadd2_rn(p, make_float2(-h.x, -h.y));
  const __half2 hh = __floats2half2_rn(h.x, h.y);
  const __half2 ll = __floats2half2_rn(l.x, l.y);
  hi = *reinterpret_cast<const uint32_t*>(&hh);
  lo = *reinterpret_cast<const uint32_t*>(&ll);
}

// the TF32 part of x as the tensor core reads it: its leading 19 bits
__device__ __forceinline__ float tf32_trunc(float x) {
  return __uint_as_float(__float_as_uint(x) & 0xffffe000u);
}

// (x0, x1) -> fp16x2 hi and lo, x = hi + lo: hi is x rounded to 11
// significant bits (exact in fp16 in its normal range), lo the rest, rounded
// to fp16; x0 goes to the low half (the lower k index of a fragment pair)
__device__ __forceinline__ void split_f16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const float h0 = tf32_rna(x0), h1 = tf32_rna(x1);
  const __half2 hh = __floats2half2_rn(h0, h1);
  const __half2 ll = __floats2half2_rn(x0 - h0, x1 - h1);
  hi = *reinterpret_cast<const uint32_t*>(&hh);
  lo = *reinterpret_cast<const uint32_t*>(&ll);
}

}  // namespace tc7

__global__ void __launch_bounds__(tc7::NT, 1)
    k_attn_tc7(TileArgs a, const __grid_constant__ CUtensorMap gmap) {
  using namespace tc7;
  extern __shared__ __align__(1024) unsigned char smem_t7[];
  unsigned char* sm = smem_t7;
  Meta& mt = *reinterpret_cast<Meta*>(sm + OFF_META);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t E = a.row_ptr[a.n_centres];
  if (E > a.capacity || (*a.status & MLG_STATUS_CAPACITY)) return;

  if (tid == 0) {
    mt.fail = 0;
    mt.nissued[0] = mt.nissued[1] = 0;
    mbar_init(&mt.bar_xfull[0], 1);
    mbar_init(&mt.bar_xfull[1], 1);
    mbar_init(&mt.bar_w, NG * GT);
    mbar_init(&mt.bar_a, NG * GT);
    mbar_init(&mt.bar_proj, 1);
    for (int h = 0; h < H; ++h) {
      mbar_init(&mt.bar_qk[h], GT);
      mbar_init(&mt.bar_s[h], 1);
      mbar_init(&mt.bar_vg[h], GT);
    }
    mbar_init(&mt.bar_fin, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&mt.tmem)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = mt.tmem;

  if (warp == 1) {
    // ------------------------------------------------------------ producer
    // The whole warp plans in step: lanes hold a window of 32 row starts
    // (the next window already loading), so a tile's plan costs shuffles, not
    // a chain of global loads; slab t lands in slot t % 2, one copy per lane,
    // once the projection of tile t - 2 (which read that slot) is done.
    const unsigned kFull = 0xffffffffu;
    int64_t c = 0, c_end = 0;
    if (lane == 0) {
      const int64_t r0 = E * blockIdx.x / gridDim.x, r1 = E * (blockIdx.x + 1) / gridDim.x;
      auto lb = [&](int64_t r) {
        int64_t lo = 0, hi = a.n_centres;
        while (lo < hi) {
          const int64_t mid = (lo + hi) >> 1;
          if (a.row_ptr[mid] < r) lo = mid + 1; else hi = mid;
        }
        return lo;
      };
      c = lb(r0);
      c_end = blockIdx.x + 1 == gridDim.x ? a.n_centres : lb(r1);
    }
    c = __shfl_sync(kFull, c, 0);
    c_end = __shfl_sync(kFull, c_end, 0);
    auto rp_at = [&](int64_t i) -> long long { return i <= a.n_centres ? a.row_ptr[i] : 0; };
    int64_t wbase = c;
    long long cur = rp_at(wbase + lane), nxt = rp_at(wbase + 31 + lane);
    const int nlim = a.nnei_max < MAXN ? a.nnei_max : MAXN;
    // plan tile t and start its slab copy into slot t % 2 (false: no tile)
    auto plan_load = [&](int t) -> bool {
      const int s = t & 1;
      Plan p;
      p.ncent = 0;
      int groups = 0;
      while (c < c_end && p.ncent < 2) {
        if (c - wbase >= 31) {   // next window (centres wbase .. wbase + 30 of each)
          wbase += 31;
          cur = nxt;
          nxt = rp_at(wbase + 31 + lane);
        }
        const int i = (int)(c - wbase);
        const long long lo = __shfl_sync(kFull, cur, i), hi = __shfl_sync(kFull, cur, i + 1);
        const int n = (int)(hi - lo);
        if (n > a.nnei_max && lane == 0) atomicOr(a.status, (uint32_t)MLG_STATUS_ROW_TOO_LONG);
        if (n < 1 || n > nlim) {  // empty, too long, or left to another kernel
          ++c;
          continue;
        }
        const int g = (n + 31) / 32;
        if (groups + g > R / 32) break;
        p.grp[p.ncent] = groups;
        p.n[p.ncent] = n;
        p.row0[p.ncent] = lo;
        ++p.ncent;
        groups += g;
        ++c;
      }
      if (lane == 0) mt.plan[t & 3] = p;
      if (p.ncent == 0) {
        if (lane == 0) mbar_arrive(&mt.bar_xfull[s]);  // no copy: the phase completes at once
        return false;
      }
      uint32_t bytes = 0;
      for (int k = 0; k < p.ncent; ++k) bytes += (uint32_t)((p.n[k] + 31) / 32) * 32 * C * 4;
      if (lane == 0) mbar_expect_tx(&mt.bar_xfull[s], bytes);
      __syncwarp();
      // copy (k, g, cc) = lane: centre k's 32-row group g, channels 4 cc .. 4 cc + 3
      {
        const int k = lane >> 4, g = (lane >> 3) & 1, cc = lane & 7;
        if (k < p.ncent && g < (p.n[k] + 31) / 32)
          tma_load_2d(sm + OFF_X + (size_t)s * A_BYTES + (size_t)cc * (R * 16) +
                          (size_t)(p.grp[k] + g) * 512,
                      &gmap, 4 * cc, (int)(p.row0[k] + 32 * g), &mt.bar_xfull[s]);
      }
      if (lane == 0) ++mt.nissued[s];
      return true;
    };
    // Tile t goes into slot t % 2 once the projection of tile t - 2 (which
    // read that slot) is done, so two tiles are planned and in flight ahead.
    Waiter wpj;
    for (int t = 0;; ++t) {
      if (t >= 2 && !wpj.wait(&mt.bar_proj)) {
        if (lane == 0) mt.fail = 1;
        break;
      }
      if (!plan_load(t)) break;
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      Waiter wa, wqk[H], ww;
      // projection of tile t: A hi is the slab as it landed (the tensor core
      // reads the TF32 part of each fp32 value, its leading 19 bits), A lo the
      // rest, x - (its leading 19 bits)
      auto issue_proj = [&](int t) {
        const uint32_t ahi = smem_u32(sm + OFF_X + (size_t)(t & 1) * A_BYTES);
        const uint32_t alo = smem_u32(sm + OFF_ALO);
        const uint32_t bhi = smem_u32(sm + OFF_WHI), blo = smem_u32(sm + OFF_WLO);
        const uint32_t id = idesc_tf32(R, N3);
#pragma unroll
        for (int s = 0; s < C / 8; ++s) {
          const uint32_t aoff = (uint32_t)(s * R * 32), boff = (uint32_t)(s * N3 * 32);
          const uint64_t dah = umma_sdesc(ahi + aoff, R * 16, 128);
          const uint64_t dal = umma_sdesc(alo + aoff, R * 16, 128);
          const uint64_t dbh = umma_sdesc(bhi + boff, N3 * 16, 128);
          const uint64_t dbl = umma_sdesc(blo + boff, N3 * 16, 128);
          umma_tf32(tmem + T_PROJ, dal, dbh, id, s > 0 ? 1u : 0u);
          umma_tf32(tmem + T_PROJ, dah, dbl, id, 1u);
          umma_tf32(tmem + T_PROJ, dah, dbh, id, 1u);
        }
        umma_commit(&mt.bar_proj);
      };
      // logits of head h: for each centre c, S[128 x nk] += Q_h^c . (K_h^c)^T,
      // nk = the tile's longest row in 16s (the key operands are zero or
      // finite past a centre's keys, and the q operands zero outside it)
      auto issue_s = [&](int h, const Plan& p) {
        int nmax = p.n[0];
        if (p.ncent > 1 && p.n[1] > nmax) nmax = p.n[1];
        const uint32_t id = idesc_tf32(R, (nmax + 15) & ~15);
        const uint32_t d = tmem + T_S + 64u * (uint32_t)h;
        for (int c = 0; c < p.ncent; ++c) {
          const uint32_t qh = tmem + T_Q + 32u * (uint32_t)h + 16u * (uint32_t)c, ql = qh + 8u;
          const uint64_t dkh = umma_sdesc(smem_u32(sm + k_off(h, c, 0)), MAXN * 16, 128);
          const uint64_t dkl = umma_sdesc(smem_u32(sm + k_off(h, c, 1)), MAXN * 16, 128);
          umma_tf32_ts(d, ql, dkh, id, c > 0 ? 1u : 0u);
          umma_tf32_ts(d, qh, dkl, id, 1u);
          umma_tf32_ts(d, qh, dkh, id, 1u);
        }
        umma_commit(&mt.bar_s[h]);
      };
      bool ok = ww.wait(&mt.bar_w) && wa.wait(&mt.bar_a);
      Plan p = mt.plan[0];
      if (ok && p.ncent > 0) {
        tc_fence_after();
        issue_proj(0);
      }
      for (int t = 0; ok && p.ncent > 0; ++t) {
        // each head's logits as soon as its group has read it back (the
        // group's read-back follows its softmax of the previous tile, so the
        // buffer is free), in the order the groups get there
        {
          uint32_t done = 0;
          const uint64_t t0 = globaltimer_ns();
          while (done != (1u << H) - 1u) {
            bool any = false;
#pragma unroll
            for (int h = 0; h < H; ++h) {
              if (!(done & (1u << h)) && mbar_test(&mt.bar_qk[h], wqk[h].par)) {
                wqk[h].par ^= 1u;
                tc_fence_after();
                issue_s(h, p);
                done |= 1u << h;
                any = true;
              }
            }
            if (!any) {
              if (globaltimer_ns() - t0 > 1000000000ull) { ok = false; break; }
              __nanosleep(32);
            }
          }
        }
        if (!ok) break;
        // the next tile's projection: every group has read this tile's back
        if (!wa.wait(&mt.bar_a)) { ok = false; break; }
        const Plan pn = mt.plan[(t + 1) & 3];
        tc_fence_after();
        if (pn.ncent > 0) issue_proj(t + 1);
        p = pn;
      }
      if (!ok) mt.fail = 1;
      // every MMA issued here is complete before TMEM is freed
      umma_commit(&mt.bar_fin);
      if (!mbar_wait(&mt.bar_fin, 0u)) mt.fail = 1;
    }
  } else {
    // ------------------------------------------------------------ compute groups
    const int grp = (warp - 2) >> 2;           // 0..3: the head of this group
    const int gtid = tid - 64;                 // 0..511 over the groups
    const int quad = warp & 3;                 // TMEM lane quadrant
    const int row = quad * 32 + lane;          // tile row of this thread
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const float qscale = (float)(1.4426950408889634 / 2.8284271247461903);  // log2(e)/sqrt(8)
    Waiter wx[2], wproj, ws, wvg;
    bool ok = true;
    // weights of the layer, split into TF32 hi / lo, K-major [96 x 32]; the
    // key operands start at zero (rows past a centre's keys stay finite)
    for (int e = gtid; e < C * N3; e += NG * GT) {
      const int k = e / N3, nn = e - k * N3;
      const int m = nn / C, cc = nn - m * C;
      const float w = static_cast<const float*>(a.W[m])[k * C + cc];
      const float hi = tf32_rna(w);
      const uint32_t off = kmajor_offset(nn, k, N3);
      *reinterpret_cast<float*>(sm + OFF_WHI + off) = hi;
      *reinterpret_cast<float*>(sm + OFF_WLO + off) = tf32_rna(w - hi);
    }
    for (int e = gtid; e < (int)(4 * H * K_BYTES / 16); e += NG * GT)
      reinterpret_cast<float4*>(sm + OFF_K)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    fence_proxy_async();
    mbar_arrive(&mt.bar_w);
    // the plan of tile t, once its slab has landed (the producer wrote the
    // plan before arming the slot)
    auto next_plan = [&](int t, Plan& p) -> bool {
      if (!wx[t & 1].wait(&mt.bar_xfull[t & 1])) return false;
      p = mt.plan[t & 3];
      return true;
    };
    // A lo of tile t (the previous projection is done with it): two float4
    // per thread, every row (a row of D depends on its own row of A only)
    auto split_lo = [&](int t, const Plan& p) {
      if (p.ncent > 0) {
        const float4* sX = reinterpret_cast<const float4*>(sm + OFF_X + (size_t)(t & 1) * A_BYTES);
        float4* sAl = reinterpret_cast<float4*>(sm + OFF_ALO);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int i = gtid + NG * GT * k;
          const float4 x = sX[i];
          sAl[i] = make_float4(x.x - tf32_trunc(x.x), x.y - tf32_trunc(x.y),
                               x.z - tf32_trunc(x.z), x.w - tf32_trunc(x.w));
        }
        fence_proxy_async();
      }
      mbar_arrive(&mt.bar_a);   // also tells the MMA thread when no work is left
    };
    // this thread's view of a tile; s of its edge is loaded here, a tile
    // ahead of its use
    auto row_info = [&](const Plan& p) -> RowInfo {
      RowInfo ri;
      ri.ncent = p.ncent;
      ri.cw = p.ncent > 0 ? centre_of_group(p, quad) : -1;
      ri.nrow = ri.cw >= 0 ? p.n[ri.cw] : 0;
      ri.key0 = ri.cw >= 0 ? 32 * p.grp[ri.cw] : 0;
      ri.vrow = ri.cw >= 0 && row - ri.key0 < ri.nrow;
      ri.orow = ri.vrow ? p.row0[ri.cw] + (row - ri.key0) : 0;
      ri.obase = ri.cw >= 0 ? p.row0[ri.cw] - ri.key0 : 0;
      ri.sw = ri.vrow ? a.sw[ri.orow] : 0.0;   // used a tile later
      return ri;
    };
    float* out = static_cast<float*>(a.out);
    const int h = grp;
    RowInfo ri;
    {
      Plan p0;
      ok = next_plan(0, p0);
      if (ok) {
        split_lo(0, p0);
        ri = row_info(p0);
      }
    }
    for (int t = 0; ok && ri.ncent > 0; ++t) {
      float* sV = reinterpret_cast<float*>(sm + OFF_V + (size_t)(t & 1) * V_BYTES);
      if (!wproj.wait(&mt.bar_proj)) { ok = false; break; }
      tc_fence_after();
      {
        // ---- read-back of head h
        uint32_t v[24];
        tmem_ld8(tmem + lane_addr + T_PROJ + 8u * h, v);
        tmem_ld8(tmem + lane_addr + T_PROJ + 32u + 8u * h, v + 8);
        tmem_ld8(tmem + lane_addr + T_PROJ + 64u + 8u * h, v + 16);
        tmem_wait_ld();
        // q (scaled by s_a log2(e)/sqrt(d)), hi and lo, into its centre's
        // TMEM operand (A of the logits), a zero row into the other's
        {
          const float fq = (float)ri.sw * qscale;
          uint32_t qv[16], zv[16];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float x = __uint_as_float(v[j]) * fq;
            const float hi = tf32_rna(x);
            qv[j] = __float_as_uint(hi);
            qv[8 + j] = __float_as_uint(tf32_rna(x - hi));
            zv[j] = zv[8 + j] = 0u;
          }
          // the warp's centre is the same for all its threads
          const uint32_t qa = tmem + lane_addr + T_Q + 32u * (uint32_t)h;
          if (ri.cw == 0) {
            tmem_st16(qa, qv);
            tmem_st16(qa + 16u, zv);
          } else if (ri.cw == 1) {
            tmem_st16(qa, zv);
            tmem_st16(qa + 16u, qv);
          } else {
            tmem_st16(qa, zv);
            tmem_st16(qa + 16u, zv);
          }
        }
        // k (scaled by s_b, kept finite) into its centre's key operand
        if (ri.cw >= 0) {
          float4 xh[2], xl[2];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float x = __uint_as_float(v[8 + j]) * (float)ri.sw;
            if (!(fabsf(x) <= 3.4028234663852886e38f)) x = 0.f;
            const float hi = tf32_rna(x);
            reinterpret_cast<float*>(xh)[j] = hi;
            reinterpret_cast<float*>(xl)[j] = tf32_rna(x - hi);
          }
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            const uint32_t off = kmajor_offset(row - ri.key0, 4 * ch, MAXN);
            *reinterpret_cast<float4*>(sm + k_off(h, ri.cw, 0) + off) = xh[ch];
            *reinterpret_cast<float4*>(sm + k_off(h, ri.cw, 1) + off) = xl[ch];
          }
        }
        // v: fp32, the two keys of a pair interleaved, [pair][head][t][key & 1]
        float* vr = sV + (row >> 1) * VS2 + h * 16 + (row & 1);
        float vm = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float x = __uint_as_float(v[16 + j]);
          vr[2 * j] = x;
          const float ax = fabsf(x);
          if (ri.vrow && ax <= 3.4028234663852886e38f) vm = fmaxf(vm, ax);   // finite, edges only
        }
        const uint32_t vb = __reduce_max_sync(0xffffffffu, __float_as_uint(vm));
        if (lane == 0) mt.vmax[h][t & 1][quad] = vb;
        fence_proxy_async();
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&mt.bar_qk[h]);
      }
      // ---- the next tile: A lo of its projection (this tile's projection
      // is done), and this thread's view of it (its s loads meanwhile)
      RowInfo rn;
      {
        Plan pn;
        if (!next_plan(t + 1, pn)) { ok = false; break; }
        split_lo(t + 1, pn);
        rn = row_info(pn);
      }
      // ---- the group's v rows of this tile in place; every thread of the
      // group is past the previous tile's softmax, so the other buffer is
      // free for the next tile
      mbar_arrive(&mt.bar_vg[h]);
      if (!wvg.wait(&mt.bar_vg[h])) { ok = false; break; }
      if (!ws.wait(&mt.bar_s[h])) { ok = false; break; }
      tc_fence_after();
      if (ri.cw >= 0) {
        // ---- head h: the logits of the warp's 32 rows over the centre's
        // keys are columns 0 .. nrow-1 of the head's buffer
        const int nrow = ri.nrow;
        const int g = lane >> 2, c = lane & 3;
        // slot-occupancy softmax: phi phantom slots of logit 0 and value 0
        const int phi = a.smooth ? a.nnei_max - nrow : 0;
        // v scale 2^-e: the tile's largest finite |v| of the head into
        // [2^13, 2^14): large values scaled down (no fp16 overflow), small
        // ones up (their lo halves stay normal in fp16)
        uint32_t vb = mt.vmax[h][t & 1][0];
#pragma unroll
        for (int w = 1; w < 4; ++w) vb = max(vb, mt.vmax[h][t & 1][w]);
        const int ev = (int)(vb >> 23) - 127;
        const int e = vb == 0 ? 0 : max(ev - 13, -110);
        const float vscale = __uint_as_float((uint32_t)(127 - e) << 23);
        const float vunscale = __uint_as_float((uint32_t)(127 + e) << 23);
        // B fragments of V_h (k = key, n = d = g), hi and lo, per 16 keys:
        // b0 = keys 16 kb + 2c, +1; b1 = keys 16 kb + 8 + 2c, +1 (keys past
        // the row are 0: they may be the other centre's rows)
        uint32_t bh[4][2], bl[4][2];
        {
          const float* vq = sV + (ri.key0 >> 1) * VS2 + h * 16 + 2 * g;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const int j = 16 * kb + 8 * hf + 2 * c;   // first key of the pair
              float2 vv = *reinterpret_cast<const float2*>(vq + (j >> 1) * VS2);
              vv.x = j < nrow ? vv.x * vscale : 0.f;
              vv.y = j + 1 < nrow ? vv.y * vscale : 0.f;
              split_f16x2(vv.x, vv.y, bh[kb][hf], bl[kb][hf]);
            }
          }
        }
        float* dst = out + h * D + 2 * c;
#pragma unroll 1
        for (int mb = 0; mb < 2; ++mb) {
          // rows ra = quad*32 + 16 mb + g and rb = ra + 8 of the tile
          const int ra = quad * 32 + 16 * mb + g;
          uint32_t sr[32];
          tmem_ld_16x256b_x8(tmem + ((uint32_t)(quad * 32 + 16 * mb) << 16) + T_S +
                                 64u * (uint32_t)h,
                             sr);
          tmem_wait_ld16(sr);
          tmem_wait_ld16(sr + 16);
          auto sf = [&](int i) { return __uint_as_float(sr[i]); };
          if (nrow < MAXN) {
            // keys past the row: logit -inf (weight 0)
#pragma unroll
            for (int k = 0; k < 8; ++k)
#pragma unroll
              for (int i = 0; i < 2; ++i)
                if (8 * k + 2 * c + i >= nrow) {
                  sr[4 * k + i] = 0xff800000u;       // -inf
                  sr[4 * k + 2 + i] = 0xff800000u;
                }
          }
          // row maxima over the quad (a tree over the thread's 16 keys)
          float m0, m1;
          {
            float t0[4], t1[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              t0[k] = fmaxf(fmaxf(sf(8 * k), sf(8 * k + 1)), fmaxf(sf(8 * k + 4), sf(8 * k + 5)));
              t1[k] = fmaxf(fmaxf(sf(8 * k + 2), sf(8 * k + 3)), fmaxf(sf(8 * k + 6), sf(8 * k + 7)));
            }
            m0 = fmaxf(fmaxf(t0[0], t0[1]), fmaxf(t0[2], t0[3]));
            m1 = fmaxf(fmaxf(t1[0], t1[1]), fmaxf(t1[2], t1[3]));
          }
          m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
          m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
          m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
          m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
          if (phi > 0) {
            m0 = fmaxf(m0, 0.f);
            m1 = fmaxf(m1, 0.f);
          }
          const float2 n0 = make_float2(-m0, -m0), n1 = make_float2(-m1, -m1);
          float2 l0 = make_float2(0.f, 0.f), l1 = make_float2(0.f, 0.f);
          // two accumulators (hi.hi and the two corrections), so that the
          // MMAs of a block of keys do not wait on one another
          float o[4] = {0.f, 0.f, 0.f, 0.f}, oc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            uint32_t ah[4], al[4];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const int k = 2 * kb + hf;
              float2 p0 = __fadd2_rn(make_float2(sf(4 * k), sf(4 * k + 1)), n0);
              float2 p1 = __fadd2_rn(make_float2(sf(4 * k + 2), sf(4 * k + 3)), n1);
              p0 = make_float2(ex2(p0.x), ex2(p0.y));
              p1 = make_float2(ex2(p1.x), ex2(p1.y));
              l0 = __fadd2_rn(l0, p0);
              l1 = __fadd2_rn(l1, p1);
              // a0a1 / a4a5: row g; a2a3 / a6a7: row g + 8
              split_p_f16x2(p0.x, p0.y, ah[2 * hf], al[2 * hf]);
              split_p_f16x2(p1.x, p1.y, ah[2 * hf + 1], al[2 * hf + 1]);
            }
            mma_f16(o, ah, bh[kb][0], bh[kb][1]);
            mma_f16(oc, ah, bl[kb][0], bl[kb][1]);
            mma_f16(oc, al, bh[kb][0], bh[kb][1]);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) o[i] += oc[i];
          float s0 = l0.x + l0.y, s1 = l1.x + l1.y;
          s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
          s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
          s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
          s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
          if (phi > 0) {
            s0 += (float)phi * ex2(-m0);
            s1 += (float)phi * ex2(-m1);
          }
          // rows g and g + 8: columns 2c, 2c + 1 of the head (8 bytes; a
          // quad writes the head's whole 32-byte sector of the row)
          if (ra - ri.key0 < nrow) {
            const float r0 = __fdividef(vunscale, s0);
            *reinterpret_cast<float2*>(dst + (ri.obase + ra) * C) = make_float2(o[0] * r0, o[1] * r0);
          }
          if (ra + 8 - ri.key0 < nrow) {
            const float r1 = __fdividef(vunscale, s1);
            *reinterpret_cast<float2*>(dst + (ri.obase + ra + 8) * C) = make_float2(o[2] * r1, o[3] * r1);
          }
        }
      }
      // the logits buffer is read: the group's next read-back arrival tells
      // the MMA thread so
      tc_fence_before();
      ri = rn;
    }
    if (!ok) mt.fail = 1;
  }
  // ---- teardown: report, let the slab copies in flight land, free TMEM
  __syncthreads();
  if (tid == 0 && mt.fail) atomicOr(a.status, kStatusTimeout);
  if (warp == 1 && lane < 2 && mt.fail && mt.nissued[lane] > 0)   // a slab copy may still land
    mbar_wait(&mt.bar_xfull[lane], (uint32_t)((mt.nissued[lane] - 1) & 1));
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

}  // namespace mlg
