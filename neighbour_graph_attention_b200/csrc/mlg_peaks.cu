// mlg_peaks.cu -- throughput microbenchmarks of the pipes the attention and
// build kernels use, on the GPU they run on (prints one JSON object).
//   fp64 FMA (DFMA), fp32 FMA (FFMA), fp64 tensor-core MMA (mma.sync f64
//   m8n8k4 and m16n8k16), the special-function pipe (ex2.approx.f32), and
//   the 5th-generation tensor cores in kind::tf32 (tcgen05.mma, M = 128, at
//   the shapes the fp32 attention issues: N = 256 as the dense reference,
//   N = 96 projection steps, N = 64 logits and N = 16 P.V steps, operand A
//   from shared memory or from TMEM).
// Each kernel runs independent dependency chains per thread so that the pipe,
// not latency, limits it; results feed a global store so nothing is removed.
//   nvcc -O3 -std=c++17 -gencode arch=compute_100a,code=sm_100a -I include \
//        -I neighbour_graph_attention_b200/csrc -o neighbour_graph_attention_b200/mlg_peaks \
//        neighbour_graph_attention_b200/csrc/mlg_peaks.cu
#include <cstdint>
#include <cstdio>
#include <cuda_runtime.h>

#include "mlg_attn_tc.cuh"

template <typename T>
__global__ void k_fma(T* out, int iters, T seed) {
  T a[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = seed + T(threadIdx.x + j);
  const T b = T(0.999999), c = T(1e-7);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int u = 0; u < 16; ++u)
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] = fma(a[j], b, c);
  }
  T s = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) s += a[j];
  if (s == T(-1)) out[blockIdx.x] = s;
}

__global__ void k_ex2(float* out, int iters) {
  float a[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = -1e-3f * (threadIdx.x + j);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int u = 0; u < 16; ++u)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float r;
        asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(a[j]));
        a[j] = r - 1.0f;
      }
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) s += a[j];
  if (s == -1.f) out[blockIdx.x] = s;
}

__global__ void k_dmma884(double* out, int iters) {
  double a = 1.0 + threadIdx.x * 1e-9, b = 0.5;
  double c[4][2];
#pragma unroll
  for (int j = 0; j < 4; ++j) c[j][0] = c[j][1] = 0.0;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        asm volatile(
            "mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
            : "+d"(c[j][0]), "+d"(c[j][1])
            : "d"(a), "d"(b));
  }
  double s = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) s += c[j][0] + c[j][1];
  if (s == -1.0) out[blockIdx.x] = s;
}

__global__ void k_dmma16816(double* out, int iters) {
  double a[8], b[4];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = 1.0 + (threadIdx.x + i) * 1e-9;
#pragma unroll
  for (int i = 0; i < 4; ++i) b[i] = 0.5;
  double c[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) c[j][i] = 0.0;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      asm volatile(
          "mma.sync.aligned.m16n8k16.row.col.f64.f64.f64.f64 {%0,%1,%2,%3}, "
          "{%4,%5,%6,%7,%8,%9,%10,%11}, {%12,%13,%14,%15}, {%0,%1,%2,%3};"
          : "+d"(c[j][0]), "+d"(c[j][1]), "+d"(c[j][2]), "+d"(c[j][3])
          : "d"(a[0]), "d"(a[1]), "d"(a[2]), "d"(a[3]), "d"(a[4]), "d"(a[5]), "d"(a[6]),
            "d"(a[7]), "d"(b[0]), "d"(b[1]), "d"(b[2]), "d"(b[3]));
  }
  double s = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) s += c[j][i];
  if (s == -1.0) out[blockIdx.x] = s;
}

__global__ void k_tf32_16816(float* out, int iters) {
  uint32_t a[4], b[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = __float_as_uint(1.0f + (threadIdx.x + i) * 1e-6f);
#pragma unroll
  for (int i = 0; i < 2; ++i) b[i] = __float_as_uint(0.5f);
  float c[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) c[j][i] = 0.f;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      asm volatile(
          "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
          "{%8,%9}, {%0,%1,%2,%3};"
          : "+f"(c[j][0]), "+f"(c[j][1]), "+f"(c[j][2]), "+f"(c[j][3])
          : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) s += c[j][i];
  if (s == -1.f) out[blockIdx.x] = s;
}

__global__ void k_bf16_16816(float* out, int iters) {
  uint32_t a[4], b[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = 0x3f803f80u + threadIdx.x;
#pragma unroll
  for (int i = 0; i < 2; ++i) b[i] = 0x3f003f00u;
  float c[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) c[j][i] = 0.f;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      asm volatile(
          "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
          "{%8,%9}, {%0,%1,%2,%3};"
          : "+f"(c[j][0]), "+f"(c[j][1]), "+f"(c[j][2]), "+f"(c[j][3])
          : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) s += c[j][i];
  if (s == -1.f) out[blockIdx.x] = s;
}

// One CTA per SM: thread 0 issues `iters` x 8 back-to-back tcgen05.mma
// kind::tf32 of M = 128, N, K = 8 into one TMEM accumulator (A from shared
// memory, or with TS from TMEM), then commits and waits (bounded).  The
// operands are small constant tiles; only the issue rate matters.
template <int N, bool TS, int NCHAIN = 1>
__global__ void __launch_bounds__(128) k_umma_tf32(float* out, int iters) {
  using namespace mlg;
  __shared__ __align__(1024) float sA[128 * 8];
  __shared__ __align__(1024) float sB[N * 8];
  __shared__ uint64_t bar;
  __shared__ uint32_t tslot;
  for (int i = threadIdx.x; i < 128 * 8; i += blockDim.x) sA[i] = 1e-3f;
  for (int i = threadIdx.x; i < N * 8; i += blockDim.x) sB[i] = 1e-3f;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tslot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  int ok = 1;
  if (threadIdx.x == 0) {
    const uint32_t id = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) |
                        ((uint32_t)(128 >> 4) << 24);
    const uint64_t da = umma_sdesc(smem_u32(sA), 128 * 16, 128);
    const uint64_t db = umma_sdesc(smem_u32(sB), N * 16, 128);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        // NCHAIN independent accumulators, used round-robin
        const uint32_t d = tmem + (uint32_t)((u % NCHAIN) * N);
        if (TS)
          asm volatile(
              "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
              "r"(tmem + 256u), "l"(db), "r"(id), "r"(1u));
        else
          umma_tf32(d, da, db, id, 1u);
      }
    }
    umma_commit(&bar);
    ok = mbar_wait(&bar, 0u) ? 1 : 0;
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
  if (threadIdx.x == 0 && !ok) out[blockIdx.x] = -1.f;
}

template <class F>
float time_ms(F launch) {
  cudaEvent_t a, b;
  cudaEventCreate(&a);
  cudaEventCreate(&b);
  launch();
  cudaDeviceSynchronize();
  float best = 1e30f;
  for (int r = 0; r < 5; ++r) {
    cudaEventRecord(a);
    launch();
    cudaEventRecord(b);
    cudaEventSynchronize(b);
    float ms = 0.f;
    cudaEventElapsedTime(&ms, a, b);
    if (ms < best) best = ms;
  }
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  return best;
}

int main() {
  int dev = 0, sms = 0, clk = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&clk, cudaDevAttrClockRate, dev);
  double* dbuf;
  float* fbuf;
  cudaMalloc(&dbuf, 1 << 20);
  cudaMalloc(&fbuf, 1 << 20);
  const int blocks = sms * 8, threads = 256, iters = 4096;
  const double lanes = (double)blocks * threads;
  float t;
  t = time_ms([&] { k_fma<double><<<blocks, threads>>>(dbuf, iters, 1.0); });
  double dfma = lanes * iters * 16 * 8 * 2 / (t * 1e-3) / 1e12;
  t = time_ms([&] { k_fma<float><<<blocks, threads>>>(fbuf, iters, 1.0f); });
  double ffma = lanes * iters * 16 * 8 * 2 / (t * 1e-3) / 1e12;
  t = time_ms([&] { k_ex2<<<blocks, threads>>>(fbuf, iters / 4); });
  double ex2 = lanes * (iters / 4) * 16 * 8 / (t * 1e-3) / 1e12;
  const double warps = (double)blocks * threads / 32;
  t = time_ms([&] { k_dmma884<<<blocks, threads>>>(dbuf, iters / 4); });
  double dmma884 = warps * (iters / 4) * 16 * (2.0 * 8 * 8 * 4) / (t * 1e-3) / 1e12;
  t = time_ms([&] { k_dmma16816<<<blocks, threads>>>(dbuf, iters / 16); });
  double dmma16816 = warps * (iters / 16) * 4 * (2.0 * 16 * 8 * 16) / (t * 1e-3) / 1e12;
  t = time_ms([&] { k_tf32_16816<<<blocks, threads>>>(fbuf, iters / 4); });
  double tf32 = warps * (iters / 4) * 4 * (2.0 * 16 * 8 * 8) / (t * 1e-3) / 1e12;
  t = time_ms([&] { k_bf16_16816<<<blocks, threads>>>(fbuf, iters / 4); });
  double bf16 = warps * (iters / 4) * 4 * (2.0 * 16 * 8 * 16) / (t * 1e-3) / 1e12;
  // tcgen05 kind::tf32: flops of M = 128, K = 8 per MMA; one CTA per SM
  const int uit = 2048;
  auto umma = [&](auto kern, int n) {
    float tt = time_ms([&] { kern<<<sms, 128>>>(fbuf, uit); });
    return (double)sms * uit * 8 * (2.0 * 128 * n * 8) / (tt * 1e-3) / 1e12;
  };
  const double u256 = umma(k_umma_tf32<256, false>, 256);
  const double u96 = umma(k_umma_tf32<96, false>, 96);
  const double u64ts = umma(k_umma_tf32<64, true>, 64);
  const double u16ts = umma(k_umma_tf32<16, true>, 16);
  // independent accumulator chains (does a short MMA pipeline across them?)
  const double u16ts4 = umma(k_umma_tf32<16, true, 4>, 16);
  const double u16ts8 = umma(k_umma_tf32<16, true, 8>, 16);
  const double u64ts4 = umma(k_umma_tf32<64, true, 4>, 64);
  const double u16ss8 = umma(k_umma_tf32<16, false, 8>, 16);
  const double u128ss2 = umma(k_umma_tf32<128, false, 2>, 128);
  cudaError_t e = cudaGetLastError();
  printf("{\"sm_count\": %d, \"clock_khz_attr\": %d, \"fp64_fma_tflops\": %.3f, "
         "\"fp32_fma_tflops\": %.3f, \"ex2_tops\": %.4f, \"dmma_m8n8k4_tflops\": %.3f, "
         "\"dmma_m16n8k16_tflops\": %.3f, \"mma_sync_tf32_m16n8k8_tflops\": %.3f, "
         "\"mma_sync_bf16_m16n8k16_tflops\": %.3f, \"tcgen05_tf32_m128n256_tflops\": %.2f, "
         "\"tcgen05_tf32_m128n96_tflops\": %.2f, \"tcgen05_tf32_ts_m128n64_tflops\": %.2f, "
         "\"tcgen05_tf32_ts_m128n16_tflops\": %.2f, \"tcgen05_tf32_ts_m128n16_4chains_tflops\": "
         "%.2f, \"tcgen05_tf32_ts_m128n16_8chains_tflops\": %.2f, "
         "\"tcgen05_tf32_ts_m128n64_4chains_tflops\": %.2f, "
         "\"tcgen05_tf32_ss_m128n16_8chains_tflops\": %.2f, "
         "\"tcgen05_tf32_ss_m128n128_2chains_tflops\": %.2f, \"cuda\": \"%s\"}\n",
         sms, clk, dfma, ffma, ex2, dmma884, dmma16816, tf32, bf16, u256, u96, u64ts, u16ts,
         u16ts4, u16ts8, u64ts4, u16ss8, u128ss2, cudaGetErrorString(e));
  cudaFree(dbuf);
  cudaFree(fbuf);
  return e == cudaSuccess ? 0 : 1;
}
