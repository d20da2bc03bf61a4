// Throughput of the pipes the scan kernels lean on, per SM and clock, on the current GPU:
// MUFU ex2 / lg2 / rcp / tanh (the "SFU" peak that bench.py divides by), FFMA and SHFL, plus
// the relative error of the approximate MUFU functions against double-precision libm.
//
// Method: every warp runs 8 independent dependency chains of one operation for many
// iterations; each CTA records clock64() at its start and end and the SM it ran on.  An SM's
// rate = (operations of the CTAs it ran) / (its last end - its first start) in SM clocks, so
// the figure does not depend on the clock the GPU happened to run at.  The mean over SMs is
// printed.
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -o bench_mufu bench_mufu.cu && ./bench_mufu
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <vector>

#define CHECK(x)                                                                     \
  do {                                                                               \
    cudaError_t e_ = (x);                                                            \
    if (e_ != cudaSuccess) {                                                         \
      std::printf("CUDA error %s at line %d\n", cudaGetErrorString(e_), __LINE__); \
      std::exit(1);                                                                  \
    }                                                                                \
  } while (0)

__device__ __forceinline__ float mufu_ex2(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float mufu_lg2(float x) {
  float y;
  asm volatile("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float mufu_rcp(float x) {
  float y;
  asm volatile("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float mufu_tanh(float x) {
  float y;
  asm volatile("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ unsigned sm_id() {
  unsigned r;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
  return r;
}

struct Span {
  long long t0, t1;
  unsigned sm, pad;
};

enum Op { kEx2, kLg2, kRcp, kTanh, kFfma, kShfl, kNumOps };
const char *kOpName[kNumOps] = {"ex2", "lg2", "rcp", "tanh", "ffma", "shfl"};

template <int OP>
__global__ void rate_kernel(float *sink, Span *spans, int iters) {
  float v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = 0.25f + 0.01f * j + 1e-6f * threadIdx.x;
  __syncthreads();
  const long long t0 = clock64();
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (OP == kEx2) v[j] = mufu_ex2(v[j]) - 1.0f;
      if (OP == kLg2) v[j] = mufu_lg2(v[j] + 1.5f);
      if (OP == kRcp) v[j] = mufu_rcp(v[j] + 1.5f);
      if (OP == kTanh) v[j] = mufu_tanh(v[j]) + 0.1f;
      if (OP == kFfma) v[j] = fmaf(v[j], 0.999f, 0.0001f);
      if (OP == kShfl) v[j] = __shfl_xor_sync(0xffffffffu, v[j], 1) * 0.999f;
    }
  }
  __syncthreads();
  const long long t1 = clock64();
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) s += v[j];
  sink[blockIdx.x * blockDim.x + threadIdx.x] = s;
  if (threadIdx.x == 0) spans[blockIdx.x] = Span{t0, t1, sm_id(), 0};
}

__global__ void accuracy_kernel(const float *x, float *ex2, float *lg2, float *rcp, float *tnh, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float a = 1.0f + fabsf(x[i]) * 0.05f;
    ex2[i] = mufu_ex2(x[i]);
    lg2[i] = mufu_lg2(a);
    rcp[i] = mufu_rcp(a);
    tnh[i] = mufu_tanh(x[i] * 0.25f);
  }
}

static double per_sm_rate(const std::vector<Span> &spans, double ops_per_cta, int nsm) {
  std::vector<long long> lo(nsm, LLONG_MAX), hi(nsm, 0);
  std::vector<int> count(nsm, 0);
  for (const Span &s : spans) {
    if (s.sm >= unsigned(nsm)) continue;
    lo[s.sm] = std::min(lo[s.sm], s.t0);
    hi[s.sm] = std::max(hi[s.sm], s.t1);
    ++count[s.sm];
  }
  double sum = 0.0;
  int used = 0;
  for (int s = 0; s < nsm; ++s)
    if (count[s]) {
      sum += ops_per_cta * count[s] / double(hi[s] - lo[s]);
      ++used;
    }
  return used ? sum / used : 0.0;
}

template <int OP>
static void measure(int nsm, float *sink, Span *spans, int blocks, int threads, int iters) {
  std::vector<Span> h(blocks);
  for (int rep = 0; rep < 2; ++rep) {  // the first launch warms up
    rate_kernel<OP><<<blocks, threads>>>(sink, spans, iters);
    CHECK(cudaDeviceSynchronize());
    CHECK(cudaGetLastError());
  }
  CHECK(cudaMemcpy(h.data(), spans, sizeof(Span) * blocks, cudaMemcpyDeviceToHost));
  std::printf("%-5s %7.2f results/clk/SM\n", kOpName[OP], per_sm_rate(h, double(threads) * iters * 8, nsm));
}

int main() {
  cudaDeviceProp prop;
  CHECK(cudaGetDeviceProperties(&prop, 0));
  const int nsm = prop.multiProcessorCount;
  std::printf("device %s, %d SMs, compute capability %d.%d\n", prop.name, nsm, prop.major, prop.minor);
  const int threads = 256, blocks = nsm * 4, iters = 4096;  // 32 warps per SM
  float *sink;
  Span *spans;
  CHECK(cudaMalloc(&sink, sizeof(float) * blocks * threads));
  CHECK(cudaMalloc(&spans, sizeof(Span) * blocks));
  measure<kEx2>(nsm, sink, spans, blocks, threads, iters);
  measure<kLg2>(nsm, sink, spans, blocks, threads, iters);
  measure<kRcp>(nsm, sink, spans, blocks, threads, iters);
  measure<kTanh>(nsm, sink, spans, blocks, threads, iters);
  measure<kFfma>(nsm, sink, spans, blocks, threads, iters);
  measure<kShfl>(nsm, sink, spans, blocks, threads, iters);

  // accuracy against libm in double precision, for the float arguments the GPU saw
  const int n = 1 << 20;
  std::vector<float> x(n);
  for (int i = 0; i < n; ++i) x[i] = -24.0f + 24.0f * float(i) / n;
  float *dx, *out[4];
  CHECK(cudaMalloc(&dx, sizeof(float) * n));
  for (float *&o : out) CHECK(cudaMalloc(&o, sizeof(float) * n));
  CHECK(cudaMemcpy(dx, x.data(), sizeof(float) * n, cudaMemcpyHostToDevice));
  accuracy_kernel<<<(n + 255) / 256, 256>>>(dx, out[0], out[1], out[2], out[3], n);
  CHECK(cudaDeviceSynchronize());
  std::vector<float> r[4];
  for (int k = 0; k < 4; ++k) {
    r[k].resize(n);
    CHECK(cudaMemcpy(r[k].data(), out[k], sizeof(float) * n, cudaMemcpyDeviceToHost));
  }
  double err[4] = {0, 0, 0, 0};
  for (int i = 0; i < n; ++i) {
    const float a = 1.0f + std::fabs(x[i]) * 0.05f;
    const double ref[4] = {std::exp2(double(x[i])), std::log2(double(a)), 1.0 / double(a),
                           std::tanh(double(x[i] * 0.25f))};
    for (int k = 0; k < 4; ++k)
      if (std::fabs(ref[k]) > 1e-3) err[k] = std::max(err[k], std::fabs(r[k][i] - ref[k]) / std::fabs(ref[k]));
  }
  std::printf("max relative error: ex2 %.3e  lg2 %.3e  rcp %.3e  tanh %.3e (|result| > 1e-3)\n", err[0], err[1],
              err[2], err[3]);
  return 0;
}
