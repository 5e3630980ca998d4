// mlg_attn_tc6.cuh -- fp32 block-dense attention, 32 channels, 4 heads of 8,
// one layer, centres of 1..64 edges: the projection and the logits on the
// 5th-generation tensor cores (tcgen05.mma kind::tf32, 3xTF32), the softmax
// and the weighted sum P V on the FP32 pipe from registers, one group of
// four warps per head that also reads back its own head's q, k and v.
//
// Per centre i with n edges (NeighborGraph issue, Proposed fix: each
// centre's edges are one small dense block, attended to with dense
// products, unequal lengths masked per row, outputs returned to the edges):
//   q_a = s_a G_a Wq log2(e)/sqrt(d),  k_b = s_b G_b Wk,  v_b = G_b Wv
//   S_ab = q_a . k_b (per head),  P_ab = 2^(S_ab - max_b S_ab),
//   O_a = sum_b P_ab v_b / sum_b P_ab.
//
// Division of the work: a tcgen05.mma of M = 128 and K = 8 takes a fixed
// ~49 cycles up to N = 64, so the contraction over a centre's keys (P V:
// eight keys per instruction, per head and per TF32 half of P) would cost far
// more on the tensor pipe than on the FP32 pipe.  The logits contract over
// d = 8: one instruction per term, head and centre.
//
// Tiles of 128 rows hold up to two centres, each starting at a multiple of
// 32 rows, so that every warp's TMEM lane quadrant belongs to one centre.
//   projection  D[128 x 96] = X[128 x 32] . [Wq|Wk|Wv], 3xTF32 (12 MMAs)
//   read-back   group h reads its head's q (scaled by s_a log2(e)/sqrt(d))
//               and k (scaled by s_b) back and splits them into TF32 hi / lo
//               K-major shared-memory operands: q into the operand of its
//               row's centre (the other centre's operand gets a zero row), k
//               into its centre's key operand at the key's slot; v as fp32
//               rows with the two keys of a pair interleaved (two buffers
//               per head, alternating between tiles)
//   logits      per head, as soon as its group has read back: for each
//               centre c, S[128 x N] += Q_h^c . (K_h^c)^T, 3 MMAs (lo.hi,
//               hi.lo, hi.hi) with N the tile's longest row in 16s.  The zero
//               rows make each centre's MMAs add exactly 0 to the other
//               centre's rows, so one buffer of N <= 64 columns holds every
//               row's logits over its own keys: each head has a buffer of
//               its own (64 columns), and a group never waits for another.
//               k is kept finite (a NaN or infinite k becomes 0) so that a
//               zero row times it stays 0; the centre still turns NaN
//               through its v.
//   group h     head h: the row's maximum from TMEM, then 16 keys at a time
//               2^(S - max) on the special-function unit, the sum, and
//               o += (p_b, p_b') . (v_b, v_b') with packed fp32x2 FMAs that
//               read both keys' values from one 16-byte load
//   output      o / sum straight to global memory: each thread's 8 values of
//               a head are one whole 32-byte sector of its output row
// A group's next read-back comes after its softmax, so its logits buffer is
// free by then: the only waits between a group and the tensor pipe are the
// projection of the next tile (issued early) and its own logits.
//
// Warp roles (576 threads, one CTA per SM):
//   warp 0      issues every MMA (one elected thread)
//   warp 1      plans tiles and loads each slab with 2-D TMA boxes of
//               {4 channels x 32 rows} straight into the K-major operand layout
//   warps 2-17  four groups of four warps, group h: the read-back of head h,
//               the split of the next slab (a quarter), the softmax of head h
// Every wait is bounded; on expiry the kernel records MLG_STATUS_TIMEOUT,
// every role leaves its loop, the MMA thread waits for its own MMAs and the
// producer for its last copy before TMEM is freed.
#pragma once

#include <cuda.h>

#include "mlg_common.cuh"
#include "mlg_attn_tile.cuh"
#include "mlg_attn_tc.cuh"
#include "mlg_attn_tc2.cuh"

namespace mlg {

namespace tc6 {

using tc2::Plan;
using tc2::Waiter;
using tc2::centre_of_group;
using tc2::ex2;
using tc2::idesc_tf32;
using tc2::mbar_arrive;

constexpr int C = 32, D = 8, H = 4, N3 = 96, R = 128;
constexpr int MAXN = 64;        // most edges of a centre handled here
constexpr int NG = 4;           // compute groups (one per head)
constexpr int GT = 128;         // threads per compute group
constexpr int NT = 64 + NG * GT;
constexpr int VS2 = 2 * C + 4;  // floats per key pair of V: [head][t][2 keys], padded

// TMEM columns (512 allocated)
constexpr uint32_t T_PROJ = 0;    // projection D: q 0-31, k 32-63, v 64-95
constexpr uint32_t T_S = 128;     // logits of head h: T_S + 64 h, [128 rows x 64 keys]

// shared memory layout (bytes)
constexpr size_t W_BYTES = (size_t)N3 * C * 4;          // one of W hi / lo (B operand)
constexpr size_t A_BYTES = (size_t)R * C * 4;           // one of X hi / lo, the raw slab
constexpr size_t Q_BYTES = (size_t)R * D * 4;           // one (head, centre) q operand, hi or lo
constexpr size_t K_BYTES = (size_t)MAXN * D * 4;        // one (head, centre) k operand, hi or lo
constexpr size_t V_BYTES = (size_t)(R / 2) * VS2 * 4;   // one V buffer
constexpr size_t OFF_WHI = 0;
constexpr size_t OFF_WLO = OFF_WHI + W_BYTES;
constexpr size_t OFF_X = OFF_WLO + W_BYTES;             // raw slab (TMA target)
constexpr size_t OFF_AHI = OFF_X + A_BYTES;
constexpr size_t OFF_ALO = OFF_AHI + A_BYTES;
constexpr size_t OFF_Q = OFF_ALO + A_BYTES;             // [head][centre][hi, lo]
constexpr size_t OFF_K = OFF_Q + 4 * H * Q_BYTES;       // [head][centre][hi, lo]
constexpr size_t OFF_V = OFF_K + 4 * H * K_BYTES;       // 2 x [64 key pairs][VS2] fp32
constexpr size_t OFF_META = OFF_V + 2 * V_BYTES;

// operand of (head h, centre c, part m: 0 hi, 1 lo)
__host__ __device__ constexpr size_t q_off(int h, int c, int m) {
  return OFF_Q + (size_t)((h * 2 + c) * 2 + m) * Q_BYTES;
}
__host__ __device__ constexpr size_t k_off(int h, int c, int m) {
  return OFF_K + (size_t)((h * 2 + c) * 2 + m) * K_BYTES;
}

struct Meta {
  Plan plan[2];             // ring of two: the tile being computed and the next
  int fail;
  uint32_t tmem;
  int last_slot;            // ring slot of the last slab copy issued (-1: none)
  uint32_t last_par;        // and the parity of the phase it completes
  uint64_t bar_xfull[2];    // slab and plan of ring slot landed (TMA tx)
  uint64_t bar_xfree;       // the groups have split the slab (count NG * GT)
  uint64_t bar_w;           // weights split, key operands zeroed (count NG * GT)
  uint64_t bar_a;           // A operands of a tile split, or no tile left (count NG * GT)
  uint64_t bar_proj;        // projection done (commit)
  uint64_t bar_qk[H];       // q and k of head h in shared memory (count GT)
  uint64_t bar_s[H];        // logits of head h done (commit)
  uint64_t bar_vg[H];       // group h has written its v rows of a tile (count GT)
  uint64_t bar_fin;         // every MMA of the CTA done (commit, at exit)
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
  bool vrow;       // the row is one of the centre's edges
  float sw;        // s of that edge (0 otherwise)
};

}  // namespace tc6

__global__ void __launch_bounds__(tc6::NT, 1)
    k_attn_tc6(TileArgs a, const __grid_constant__ CUtensorMap gmap) {
  using namespace tc6;
  extern __shared__ __align__(1024) unsigned char smem_t6[];
  unsigned char* sm = smem_t6;
  Meta& mt = *reinterpret_cast<Meta*>(sm + OFF_META);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t E = a.row_ptr[a.n_centres];
  if (E > a.capacity || (*a.status & MLG_STATUS_CAPACITY)) return;

  if (tid == 0) {
    mt.fail = 0;
    mt.last_slot = -1;
    mt.last_par = 0;
    mbar_init(&mt.bar_xfull[0], 1);
    mbar_init(&mt.bar_xfull[1], 1);
    mbar_init(&mt.bar_xfree, NG * GT);
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
      int64_t c = lb(r0);
      const int64_t c_end = blockIdx.x + 1 == gridDim.x ? a.n_centres : lb(r1);
      const int nlim = a.nnei_max < MAXN ? a.nnei_max : MAXN;
      Waiter wfree;
      for (int t = 0;; ++t) {
        const int s = t & 1;
        if (t > 0 && !wfree.wait(&mt.bar_xfree)) {  // the previous slab was split
          mt.fail = 1;
          break;
        }
        Plan p;
        p.ncent = 0;
        int groups = 0;
        while (c < c_end && p.ncent < 2) {
          const int n = (int)(a.row_ptr[c + 1] - a.row_ptr[c]);
          if (n > a.nnei_max) atomicOr(a.status, (uint32_t)MLG_STATUS_ROW_TOO_LONG);
          if (n < 1 || n > nlim) {  // empty, too long, or left to another kernel
            ++c;
            continue;
          }
          const int g = (n + 31) / 32;
          if (groups + g > R / 32) break;
          p.grp[p.ncent] = groups;
          p.n[p.ncent] = n;
          p.row0[p.ncent] = a.row_ptr[c];
          ++p.ncent;
          groups += g;
          ++c;
        }
        mt.plan[s] = p;
        if (p.ncent == 0) {
          mbar_arrive(&mt.bar_xfull[s]);  // no copy: the phase completes at once
          break;
        }
        fence_proxy_async();
        uint32_t bytes = 0;
        for (int k = 0; k < p.ncent; ++k) bytes += (uint32_t)((p.n[k] + 31) / 32) * 32 * C * 4;
        mbar_expect_tx(&mt.bar_xfull[s], bytes);
        for (int k = 0; k < p.ncent; ++k)
          for (int g = 0; g < (p.n[k] + 31) / 32; ++g)
            for (int cc = 0; cc < C / 4; ++cc)
              tma_load_2d(sm + OFF_X + (size_t)cc * (R * 16) + (size_t)(p.grp[k] + g) * 512,
                          &gmap, 4 * cc, (int)(p.row0[k] + 32 * g), &mt.bar_xfull[s]);
        mt.last_slot = s;
        mt.last_par = (uint32_t)((t >> 1) & 1);  // the phase of slot s this copy completes
      }
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      Waiter wa, wqk[H], ww;
      auto issue_proj = [&]() {
        const uint32_t ahi = smem_u32(sm + OFF_AHI), alo = smem_u32(sm + OFF_ALO);
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
          const uint64_t dqh = umma_sdesc(smem_u32(sm + q_off(h, c, 0)), R * 16, 128);
          const uint64_t dql = umma_sdesc(smem_u32(sm + q_off(h, c, 1)), R * 16, 128);
          const uint64_t dkh = umma_sdesc(smem_u32(sm + k_off(h, c, 0)), MAXN * 16, 128);
          const uint64_t dkl = umma_sdesc(smem_u32(sm + k_off(h, c, 1)), MAXN * 16, 128);
          umma_tf32(d, dql, dkh, id, c > 0 ? 1u : 0u);
          umma_tf32(d, dqh, dkl, id, 1u);
          umma_tf32(d, dqh, dkh, id, 1u);
        }
        umma_commit(&mt.bar_s[h]);
      };
      bool ok = ww.wait(&mt.bar_w) && wa.wait(&mt.bar_a);
      Plan p = mt.plan[0];
      if (ok && p.ncent > 0) {
        tc_fence_after();
        issue_proj();
      }
      for (int t = 0; ok && p.ncent > 0; ++t) {
        // head h as soon as group h has read it back (the group's read-back
        // follows its softmax of the previous tile, so the buffer is free)
#pragma unroll
        for (int h = 0; h < H; ++h) {
          if (!ok) break;
          ok = wqk[h].wait(&mt.bar_qk[h]);
          if (!ok) break;
          tc_fence_after();
          issue_s(h, p);
        }
        if (!ok) break;
        // the next tile's projection: every group has read this tile's back
        if (!wa.wait(&mt.bar_a)) { ok = false; break; }
        const Plan pn = mt.plan[(t + 1) & 1];
        tc_fence_after();
        if (pn.ncent > 0) issue_proj();
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
    // The slab of ring slot s split into the A operands (rows outside the
    // centres are 0).  Thread gtid takes the 8 elements e = gtid + 512 k,
    // k = 0..7: in the K-major layout (128-byte core matrices, 16 row groups
    // per 4-element K chunk) these are column 4 k + (gtid & 3) of one row.
    const int r0 = (gtid >> 5) * 8 + ((gtid & 31) >> 2);
    auto split = [&](int s, Plan& p) -> bool {
      if (!wx[s].wait(&mt.bar_xfull[s])) return false;
      p = mt.plan[s];
      if (p.ncent > 0) {
        const float* sX = reinterpret_cast<const float*>(sm + OFF_X);
        float* sAh = reinterpret_cast<float*>(sm + OFF_AHI);
        float* sAl = reinterpret_cast<float*>(sm + OFF_ALO);
        const int cg = centre_of_group(p, r0 >> 5);
        const bool valid = cg >= 0 && r0 - 32 * p.grp[cg] < p.n[cg];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int e = gtid + NG * GT * k;
          const float x = valid ? sX[e] : 0.f;
          const float hi = tf32_rna(x);
          sAh[e] = hi;
          sAl[e] = tf32_rna(x - hi);
        }
        fence_proxy_async();
        mbar_arrive(&mt.bar_xfree);
      }
      mbar_arrive(&mt.bar_a);  // also tells the MMA thread when no work is left
      return true;
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
      ri.sw = ri.vrow ? (float)a.sw[ri.orow] : 0.f;
      return ri;
    };
    float* out = static_cast<float*>(a.out);
    const int h = grp;
    RowInfo ri;
    {
      Plan p0;
      ok = split(0, p0);
      ri = row_info(p0);
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
        // q (scaled by s_a log2(e)/sqrt(d)) into its centre's operand, a zero
        // row into the other's
        {
          const float fq = ri.sw * qscale;
          float4 xh[2], xl[2];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float x = __uint_as_float(v[j]) * fq;
            const float hi = tf32_rna(x);
            reinterpret_cast<float*>(xh)[j] = hi;
            reinterpret_cast<float*>(xl)[j] = tf32_rna(x - hi);
          }
          const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const bool mine = c == ri.cw;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
              const uint32_t off = kmajor_offset(row, 4 * ch, R);
              *reinterpret_cast<float4*>(sm + q_off(h, c, 0) + off) = mine ? xh[ch] : z;
              *reinterpret_cast<float4*>(sm + q_off(h, c, 1) + off) = mine ? xl[ch] : z;
            }
          }
        }
        // k (scaled by s_b, kept finite) into its centre's key operand
        if (ri.cw >= 0) {
          float4 xh[2], xl[2];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float x = __uint_as_float(v[8 + j]) * ri.sw;
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
#pragma unroll
        for (int j = 0; j < 8; ++j) vr[2 * j] = __uint_as_float(v[16 + j]);
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(&mt.bar_qk[h]);
      }
      // ---- the next tile's slab into the A operands (its projection then
      // overlaps this tile's softmax), and this thread's view of it
      RowInfo rn;
      {
        Plan pn;
        if (!split((t + 1) & 1, pn)) { ok = false; break; }
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
        // ---- head h: the row's logits over its own keys are columns
        // 0 .. nrow-1 of the head's buffer
        const int nrow = ri.nrow;
        const uint32_t sa = tmem + lane_addr + T_S + 64u * (uint32_t)h;
        // slot-occupancy softmax: phi phantom slots of logit 0 and value 0
        const int phi = a.smooth ? a.nnei_max - nrow : 0;
        float mx;
        float2 ls = make_float2(0.f, 0.f);
        float2 acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = make_float2(0.f, 0.f);
        const float* vp = sV + (ri.key0 >> 1) * VS2 + h * 16;
        if (nrow == MAXN) {
          // ---- full rows (the common case), no per-key masks, two passes
          // over the row in TMEM: its maximum, then 16 keys at a time (the
          // next 16 loading while these are used) 2^(S - max), the sum and P V
          {
            uint32_t sr[64];
            tmem_ld16(sa, sr);
            tmem_ld16(sa + 16u, sr + 16);
            tmem_ld16(sa + 32u, sr + 32);
            tmem_ld16(sa + 48u, sr + 48);
            tmem_wait_ld16(sr);
            tmem_wait_ld16(sr + 16);
            tmem_wait_ld16(sr + 32);
            tmem_wait_ld16(sr + 48);
            float m4[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              m4[c] = __uint_as_float(sr[16 * c]);
#pragma unroll
              for (int j = 1; j < 16; ++j) m4[c] = fmaxf(m4[c], __uint_as_float(sr[16 * c + j]));
            }
            mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            if (phi > 0) mx = fmaxf(mx, 0.f);
          }
          const float2 m2 = make_float2(-mx, -mx);
          uint32_t sq[2][16];
          tmem_ld16(sa, sq[0]);
          tmem_wait_ld16(sq[0]);
#pragma unroll
          for (int qt = 0; qt < 4; ++qt) {
            uint32_t* cur = sq[qt & 1];
            if (qt < 3) tmem_ld16(sa + 16u * (uint32_t)(qt + 1), sq[(qt + 1) & 1]);
#pragma unroll
            for (int jp = 0; jp < 8; ++jp) {
              float2 p2 = __fadd2_rn(
                  make_float2(__uint_as_float(cur[2 * jp]), __uint_as_float(cur[2 * jp + 1])), m2);
              p2 = make_float2(ex2(p2.x), ex2(p2.y));
              ls = __fadd2_rn(ls, p2);
              const float4* v4 = reinterpret_cast<const float4*>(vp + (8 * qt + jp) * VS2);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float4 w = v4[q];
                acc[2 * q] = __ffma2_rn(p2, make_float2(w.x, w.y), acc[2 * q]);
                acc[2 * q + 1] = __ffma2_rn(p2, make_float2(w.z, w.w), acc[2 * q + 1]);
              }
            }
            if (qt < 3) tmem_wait_ld16(sq[(qt + 1) & 1]);
          }
        } else {
          // ---- ragged rows (1..63 edges, the same for every thread of the
          // warp): the same two passes, 16 keys per load, keys past the row
          // masked (the odd key of a row's last pair is a zero padding row)
          const int nq = (nrow + 15) >> 4;
          float m = phi > 0 ? 0.f : -INFINITY;
#pragma unroll 1
          for (int qt = 0; qt < nq; ++qt) {
            uint32_t sr[16];
            tmem_ld16(sa + 16u * (uint32_t)qt, sr);
            tmem_wait_ld16(sr);
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (16 * qt + j < nrow) m = fmaxf(m, __uint_as_float(sr[j]));
          }
          mx = m;
          const float2 m2 = make_float2(-mx, -mx);
#pragma unroll 1
          for (int qt = 0; qt < nq; ++qt) {
            uint32_t sr[16];
            tmem_ld16(sa + 16u * (uint32_t)qt, sr);
            tmem_wait_ld16(sr);
#pragma unroll
            for (int jp = 0; jp < 8; ++jp) {
              const int kk = 16 * qt + 2 * jp;
              if (kk < nrow) {
                float2 p2 = __fadd2_rn(
                    make_float2(__uint_as_float(sr[2 * jp]), __uint_as_float(sr[2 * jp + 1])), m2);
                p2 = make_float2(ex2(p2.x), kk + 1 < nrow ? ex2(p2.y) : 0.f);
                ls = __fadd2_rn(ls, p2);
                const float4* v4 = reinterpret_cast<const float4*>(vp + (kk / 2) * VS2);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const float4 w = v4[q];  // (v_b[t], v_b'[t], v_b[t+1], v_b'[t+1]), t = 2 q
                  acc[2 * q] = __ffma2_rn(p2, make_float2(w.x, w.y), acc[2 * q]);
                  acc[2 * q + 1] = __ffma2_rn(p2, make_float2(w.z, w.w), acc[2 * q + 1]);
                }
              }
            }
          }
        }
        const float l = (ls.x + ls.y) + (phi > 0 ? (float)phi * ex2(-mx) : 0.f);
        if (ri.vrow) {
          // one whole 32-byte sector of the output row
          const float rl = 1.f / l;
          float* dst = out + ri.orow * C + h * D;
          *reinterpret_cast<float4*>(dst) =
              make_float4((acc[0].x + acc[0].y) * rl, (acc[1].x + acc[1].y) * rl,
                          (acc[2].x + acc[2].y) * rl, (acc[3].x + acc[3].y) * rl);
          *reinterpret_cast<float4*>(dst + 4) =
              make_float4((acc[4].x + acc[4].y) * rl, (acc[5].x + acc[5].y) * rl,
                          (acc[6].x + acc[6].y) * rl, (acc[7].x + acc[7].y) * rl);
        }
      }
      // the logits buffer is read: the group's next read-back arrival tells
      // the MMA thread so
      tc_fence_before();
      ri = rn;
    }
    if (!ok) mt.fail = 1;
  }
  // ---- teardown: report, let a slab copy in flight land, free TMEM
  __syncthreads();
  if (tid == 0 && mt.fail) atomicOr(a.status, kStatusTimeout);
  if (warp == 1 && lane == 0 && mt.fail && mt.last_slot >= 0)
    mbar_wait(&mt.bar_xfull[mt.last_slot], mt.last_par);  // a slab copy may still land
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

}  // namespace mlg
