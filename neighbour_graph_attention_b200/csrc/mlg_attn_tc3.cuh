// mlg_attn_tc3.cuh -- fp32 block-dense attention, 32 channels, 4 heads of 8,
// one layer, centres of 1..64 edges: the projection and the logits on the
// 5th-generation tensor cores (tcgen05.mma kind::tf32, 3xTF32), the softmax
// and the weighted sum P V on the FP32 pipe from registers.
//
// Per centre i with n edges (NeighborGraph issue, Proposed fix: each
// centre's edges are one small dense block, attended to with dense
// products, unequal lengths masked per row, outputs returned to the edges):
//   q_a = s_a G_a Wq log2(e)/sqrt(d),  k_b = s_b G_b Wk,  v_b = G_b Wv
//   S_ab = q_a . k_b (per head),  P_ab = 2^(S_ab - max_b S_ab),
//   O_a = sum_b P_ab v_b / sum_b P_ab.
//
// Why the split between the units: a tcgen05.mma of M = 128 and K = 8 costs
// a fixed number of cycles for small N (measured: N = 16 and N = 64 run at
// the same rate per instruction), and P V contracts over the keys, eight per
// instruction, for every head and for P's two TF32 halves: 128 instructions
// per tile of two centres.  The logits contract over d = 8 only: one
// instruction per term and head, N = 128 covering both centres' keys at once
// (the blocks between different centres are computed and never read).
//
// Tiles of 128 rows hold up to two centres, each starting at a multiple of
// 32 rows, so that every warp's TMEM lane quadrant belongs to one centre.
//   projection  D[128 x 96] = X[128 x 32] . [Wq|Wk|Wv], 3xTF32 (12 MMAs)
//   Q, K        read back, scaled, split into TF32 hi / lo: shared-memory
//               operands of the logits; V read back as fp32 rows
//   logits      per head: S[128 x 128] = Q_h . K_h^T, 3 MMAs (lo.hi, hi.lo,
//               hi.hi) into one of two TMEM buffers
//   softmax     one thread per row: its centre's S columns from TMEM into
//               registers (the buffer is released at once), max, 2^(S - max)
//               on the special-function unit, sum
//   P V         o = sum_b p_b v_b with broadcast reads of the centre's v_b
//               rows, packed fp32x2 FMAs
//   output      o / sum straight to global memory: each thread's 8 values of
//               a head are one whole 32-byte sector of its output row
// The projection's TMEM is free once Q, K and V are read back, so the next
// slab is split at once and its projection runs during this tile's softmax.
//
// Warp roles (320 threads, one CTA per SM):
//   warp 0     issues every MMA (one elected thread)
//   warp 1     plans tiles and loads each slab with 2-D TMA boxes of
//              {4 channels x 32 rows} straight into the K-major operand layout
//   warps 2-5  group 0: split, Q and K, heads 0 and 2
//   warps 6-9  group 1: split, V, heads 1 and 3
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

namespace tc3 {

using tc2::Plan;
using tc2::Waiter;
using tc2::centre_of_group;
using tc2::ex2;
using tc2::idesc_tf32;
using tc2::mbar_arrive;

constexpr int C = 32, D = 8, H = 4, N3 = 96, R = 128;
constexpr int MAXN = 64;        // most edges of a centre handled here
constexpr int NT = 320;         // threads
constexpr int GT = 128;         // threads per compute group
constexpr int VS = C + 4;       // V row stride (floats): conflict-free 16-byte row stores

// TMEM columns (512 allocated)
constexpr uint32_t T_PROJ = 0;    // projection D: q 0-31, k 32-63, v 64-95
constexpr uint32_t T_S = 128;     // logits buffer b: T_S + 128 b, [128 rows x 128 keys]

// shared memory layout (bytes)
constexpr size_t W_BYTES = (size_t)N3 * C * 4;          // one of W hi / lo (B operand)
constexpr size_t A_BYTES = (size_t)R * C * 4;           // one of X hi / lo, the raw slab
constexpr size_t K_BYTES = (size_t)R * D * 4;           // one head of Q or K, hi or lo
constexpr size_t OFF_WHI = 0;
constexpr size_t OFF_WLO = OFF_WHI + W_BYTES;
constexpr size_t OFF_X = OFF_WLO + W_BYTES;             // raw slab (TMA target)
constexpr size_t OFF_AHI = OFF_X + A_BYTES;
constexpr size_t OFF_ALO = OFF_AHI + A_BYTES;
constexpr size_t OFF_Q = OFF_ALO + A_BYTES;             // [head][hi, lo]
constexpr size_t OFF_K = OFF_Q + 2 * H * K_BYTES;       // [head][hi, lo]
constexpr size_t OFF_V = OFF_K + 2 * H * K_BYTES;       // [128][VS] fp32
constexpr size_t OFF_META = OFF_V + (size_t)R * VS * 4;

struct Meta {
  Plan plan[2];             // ring of two: the tile being computed and the next
  int fail;
  uint32_t tmem;
  int last_slot;            // ring slot of the last slab copy issued (-1: none)
  uint32_t last_par;        // and the parity of the phase it completes
  uint64_t bar_xfull[2];    // slab and plan of ring slot landed (TMA tx)
  uint64_t bar_xfree;       // the groups have split the slab (count 2 * GT)
  uint64_t bar_w;           // weights split (count 2 * GT)
  uint64_t bar_a;           // A operands of a tile split, or no tile left (count 2 * GT)
  uint64_t bar_proj;        // projection done (commit)
  uint64_t bar_qk;          // Q and K in shared memory (count GT)
  uint64_t bar_v;           // V rows in shared memory (count GT)
  uint64_t bar_s[2];        // logits of buffer b done (commit)
  uint64_t bar_sfree[2];    // logits of buffer b read into registers (count GT)
  uint64_t bar_vfree;       // both groups are done with the V rows of a tile (count 2 * GT)
  uint64_t bar_fin;         // every MMA of the CTA done (commit, at exit)
};
constexpr size_t SMEM = OFF_META + sizeof(Meta);
static_assert(SMEM <= 227 * 1024, "shared memory");
static_assert(SMEM > 116 * 1024, "one CTA per SM (the kernel holds all 512 TMEM columns)");

}  // namespace tc3

__global__ void __launch_bounds__(tc3::NT, 1)
    k_attn_tc3(TileArgs a, const __grid_constant__ CUtensorMap gmap) {
  using namespace tc3;
  extern __shared__ __align__(1024) unsigned char smem_t3[];
  unsigned char* sm = smem_t3;
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
    mbar_init(&mt.bar_xfree, 2 * GT);
    mbar_init(&mt.bar_w, 2 * GT);
    mbar_init(&mt.bar_a, 2 * GT);
    mbar_init(&mt.bar_proj, 1);
    mbar_init(&mt.bar_qk, GT);
    mbar_init(&mt.bar_v, GT);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&mt.bar_s[b], 1);
      mbar_init(&mt.bar_sfree[b], GT);
    }
    mbar_init(&mt.bar_vfree, 2 * GT);
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
      Waiter wa, wqk, wsf[2], ww;
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
      // logits of head h over all keys of the tile: S[128 x nk] = Q_h . K_h^T
      auto issue_s = [&](int h, int b, int nk) {
        const uint32_t qhi = smem_u32(sm + OFF_Q + (size_t)(2 * h) * K_BYTES);
        const uint32_t khi = smem_u32(sm + OFF_K + (size_t)(2 * h) * K_BYTES);
        const uint64_t dqh = umma_sdesc(qhi, R * 16, 128);
        const uint64_t dql = umma_sdesc(qhi + (uint32_t)K_BYTES, R * 16, 128);
        const uint64_t dkh = umma_sdesc(khi, R * 16, 128);
        const uint64_t dkl = umma_sdesc(khi + (uint32_t)K_BYTES, R * 16, 128);
        const uint32_t id = idesc_tf32(R, nk);
        const uint32_t d = tmem + T_S + 128u * b;
        umma_tf32(d, dql, dkh, id, 0u);
        umma_tf32(d, dqh, dkl, id, 1u);
        umma_tf32(d, dqh, dkh, id, 1u);
        umma_commit(&mt.bar_s[b]);
      };
      bool ok = ww.wait(&mt.bar_w) && wa.wait(&mt.bar_a);
      Plan p = mt.plan[0];
      if (ok && p.ncent > 0) {
        tc_fence_after();
        issue_proj();
      }
      for (int t = 0; ok && p.ncent > 0; ++t) {
        // keys of the tile: up to the end of the last centre's 32-row groups, in 16s
        const int last = p.ncent - 1;
        const int nk = (32 * p.grp[last] + p.n[last] + 15) & ~15;
        if (!wqk.wait(&mt.bar_qk)) { ok = false; break; }
        tc_fence_after();
        // both buffers were read out by the previous tile's last two heads
        if (t > 0 && (!wsf[0].wait(&mt.bar_sfree[0]) || !wsf[1].wait(&mt.bar_sfree[1]))) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_s(0, 0, nk);
        issue_s(1, 1, nk);
        // heads 2 and 3 once the groups have read heads 0 and 1 out
        for (int b = 0; b < 2 && ok; ++b) {
          if (!wsf[b].wait(&mt.bar_sfree[b])) { ok = false; break; }
          tc_fence_after();
          issue_s(b + 2, b, nk);
        }
        if (!ok) break;
        // the groups have read the projection out of TMEM: the next tile's
        // projection runs on the tensor cores during the rest of this tile's
        // softmax.  Its commit follows every logits MMA of this tile, so the
        // groups' wait for it also tells them Q and K may be overwritten.
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
    const int grp = (warp - 2) >> 2;           // 0 or 1
    const int quad = warp & 3;                 // TMEM lane quadrant
    const int row = quad * 32 + lane;          // tile row of this thread
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const float qscale = (float)(1.4426950408889634 / 2.8284271247461903);  // log2(e)/sqrt(8)
    Waiter wx[2], wproj, ws[2], wv, wvf;
    bool ok = true;
    // weights of the layer, split into TF32 hi / lo, K-major [96 x 32]
    for (int e = tid - 64; e < C * N3; e += 2 * GT) {
      const int k = e / N3, nn = e - k * N3;
      const int m = nn / C, cc = nn - m * C;
      const float w = static_cast<const float*>(a.W[m])[k * C + cc];
      const float hi = tf32_rna(w);
      const uint32_t off = kmajor_offset(nn, k, N3);
      *reinterpret_cast<float*>(sm + OFF_WHI + off) = hi;
      *reinterpret_cast<float*>(sm + OFF_WLO + off) = tf32_rna(w - hi);
    }
    fence_proxy_async();
    mbar_arrive(&mt.bar_w);
    // the slab of ring slot s split into the A operands (rows outside the
    // centres are 0); returns the slot's plan (ncent 0: no work left)
    auto split = [&](int s, Plan& p) -> bool {
      if (!wx[s].wait(&mt.bar_xfull[s])) return false;
      p = mt.plan[s];
      if (p.ncent > 0) {
        const float* sX = reinterpret_cast<const float*>(sm + OFF_X);
        float* sAh = reinterpret_cast<float*>(sm + OFF_AHI);
        float* sAl = reinterpret_cast<float*>(sm + OFF_ALO);
        for (int e = tid - 64; e < R * C; e += 2 * GT) {
          const int core = e >> 5, w = e & 31;
          const int r = (core % (R / 8)) * 8 + (w >> 2);
          const int cg = centre_of_group(p, r >> 5);
          const bool valid = cg >= 0 && r - 32 * p.grp[cg] < p.n[cg];
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
    const float* sV = reinterpret_cast<const float*>(sm + OFF_V);
    float* out = static_cast<float*>(a.out);
    Plan p;
    ok = split(0, p);
    for (int t = 0; ok && p.ncent > 0; ++t) {
      const int cw = centre_of_group(p, quad);   // this warp's centre (-1: none)
      const int nrow = cw >= 0 ? p.n[cw] : 0;
      const int key0 = cw >= 0 ? 32 * p.grp[cw] : 0;  // the centre's first key (tile row)
      const bool vrow = cw >= 0 && row - key0 < nrow;
      if (!wproj.wait(&mt.bar_proj)) { ok = false; break; }
      tc_fence_after();
      if (grp == 0) {
        // ---- Q (scaled by s_a log2(e)/sqrt(d)) and K (scaled by s_b), split,
        // K-major shared-memory operands of the logits
        const float sw = vrow ? (float)a.sw[p.row0[cw] + (row - key0)] : 0.f;
        uint32_t v[16];
#pragma unroll
        for (int part = 0; part < 4; ++part) {
          tmem_ld16(tmem + lane_addr + T_PROJ + 16u * part, v);
          tmem_wait_ld();
          const float f = part < 2 ? sw * qscale : sw;
          unsigned char* base = sm + (part < 2 ? OFF_Q : OFF_K);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int h = 2 * (part & 1) + hh;
            float4 xh[2], xl[2];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float x = __uint_as_float(v[8 * hh + j]) * f;
              const float hi = tf32_rna(x);
              reinterpret_cast<float*>(xh)[j] = hi;
              reinterpret_cast<float*>(xl)[j] = tf32_rna(x - hi);
            }
            unsigned char* hb = base + (size_t)(2 * h) * K_BYTES;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
              const uint32_t off = kmajor_offset(row, 4 * ch, R);
              *reinterpret_cast<float4*>(hb + off) = xh[ch];
              *reinterpret_cast<float4*>(hb + K_BYTES + off) = xl[ch];
            }
          }
        }
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(&mt.bar_qk);
      } else {
        // ---- V rows, fp32 (padded stride: conflict-free 16-byte stores), once
        // group 0 is done with the previous tile's rows
        if (t > 0 && !wvf.wait(&mt.bar_vfree)) { ok = false; break; }
        uint32_t v[16];
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          tmem_ld16(tmem + lane_addr + T_PROJ + 64u + 16u * part, v);
          tmem_wait_ld();
          float* vr = const_cast<float*>(sV) + row * VS + 16 * part;
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            *reinterpret_cast<float4*>(vr + j) =
                make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                            __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
        }
        tc_fence_before();
        mbar_arrive(&mt.bar_v);
      }
      // ---- the next tile's slab into the A operands (its projection then
      // overlaps this tile's softmax)
      Plan pn;
      if (!split((t + 1) & 1, pn)) { ok = false; break; }
      // ---- V rows of this tile must be in place (group 1 wrote them)
      if (!wv.wait(&mt.bar_v)) { ok = false; break; }
      // ---- heads grp and grp + 2: softmax and P V from registers
      const int b = grp;
      for (int hi2 = 0; hi2 < 2 && ok; ++hi2) {
        const int h = grp + 2 * hi2;
        if (!ws[b].wait(&mt.bar_s[b])) { ok = false; break; }
        tc_fence_after();
        float sv[MAXN];
        const int nn = (nrow + 15) & ~15;
        if (cw >= 0) {
          uint32_t v[16];
#pragma unroll
          for (int q = 0; q < MAXN / 16; ++q) {
            if (16 * q < nn) {
              tmem_ld16(tmem + lane_addr + T_S + 128u * b + (uint32_t)key0 + 16u * q, v);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 16; ++j) sv[16 * q + j] = __uint_as_float(v[j]);
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) sv[16 * q + j] = -INFINITY;
            }
          }
        }
        // the logits are in registers: the buffer can take the next head's
        tc_fence_before();
        mbar_arrive(&mt.bar_sfree[b]);
        if (cw >= 0) {
          float mx = -INFINITY;
#pragma unroll
          for (int j = 0; j < MAXN; ++j) {
            if (j >= nrow) sv[j] = -INFINITY;
            mx = fmaxf(mx, sv[j]);
          }
          // slot-occupancy softmax: phi phantom slots of logit 0 and value 0
          const int phi = a.smooth ? a.nnei_max - nrow : 0;
          if (phi > 0) mx = fmaxf(mx, 0.f);
          if (!vrow) mx = 0.f;
          float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
#pragma unroll
          for (int j = 0; j < MAXN; j += 4) {
            sv[j] = ex2(sv[j] - mx);
            sv[j + 1] = ex2(sv[j + 1] - mx);
            sv[j + 2] = ex2(sv[j + 2] - mx);
            sv[j + 3] = ex2(sv[j + 3] - mx);
            l0 += sv[j];
            l1 += sv[j + 1];
            l2 += sv[j + 2];
            l3 += sv[j + 3];
          }
          const float l = (l0 + l1) + (l2 + l3) + (phi > 0 ? (float)phi * ex2(-mx) : 0.f);
          // o = sum_b p_b v_b over the centre's keys (broadcast reads of v_b)
          float2 o[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
          const float* vb = sV + key0 * VS + h * D;
#pragma unroll
          for (int j = 0; j < MAXN; ++j) {
            if (j < nrow) {
              const float4 v0 = *reinterpret_cast<const float4*>(vb + j * VS);
              const float4 v1 = *reinterpret_cast<const float4*>(vb + j * VS + 4);
              const float2 pj = make_float2(sv[j], sv[j]);
              o[0] = __ffma2_rn(pj, make_float2(v0.x, v0.y), o[0]);
              o[1] = __ffma2_rn(pj, make_float2(v0.z, v0.w), o[1]);
              o[2] = __ffma2_rn(pj, make_float2(v1.x, v1.y), o[2]);
              o[3] = __ffma2_rn(pj, make_float2(v1.z, v1.w), o[3]);
            }
          }
          if (vrow) {
            // one whole 32-byte sector of the output row
            const float rl = 1.f / l;
            float* dst = out + (p.row0[cw] + (row - key0)) * C + h * D;
            *reinterpret_cast<float4*>(dst) =
                make_float4(o[0].x * rl, o[0].y * rl, o[1].x * rl, o[1].y * rl);
            *reinterpret_cast<float4*>(dst + 4) =
                make_float4(o[2].x * rl, o[2].y * rl, o[3].x * rl, o[3].y * rl);
          }
        }
      }
      if (!ok) break;
      // this group is done with the tile's V rows
      mbar_arrive(&mt.bar_vfree);
      p = pn;
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
