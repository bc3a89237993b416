// Issue cost and throughput of tcgen05.mma (kind::f16, bf16 operands, fp32
// accumulator in TMEM) by shape and by how the issuing code is written.
//
// Each CTA holds an A tile [M x 64] and a B tile [N x 64] (K-major, 128-byte
// swizzle, zero-filled) in shared memory and a TMEM accumulator. ITERS groups
// of four MMAs (K = 64) are issued back to back; each group is committed to an
// mbarrier, and before issuing group i the code waits for the commit of group
// i - 2 (bounded by %globaltimer). Reported per case: TFLOP/s, cycles per MMA
// per SM, and the cycles spent issuing one group (clock64 around the issue).
//
// Issue modes:
//   0  one thread (a lane-0 branch), one asm statement per MMA with its own
//      accumulate predicate, then the commit;
//   1  the whole warp runs the loop; each MMA and the commit are guarded by
//      elect.sync inside their own asm statement;
//   2  the whole warp runs the loop; one asm block elects once and issues the
//      four MMAs (immediate accumulate predicates) and the commit.
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 -o mma_issue mma_issue.cu && ./mma_issue
//
// Shared memory per CTA is 49 KB and TMEM 128 columns, so 4 CTAs fit on an SM.
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>

__device__ __forceinline__ uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint64_t desc_k(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)(16 >> 4) << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
__host__ __device__ constexpr uint32_t idesc(uint32_t m, uint32_t n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((m >> 4) << 24);
}
__device__ __forceinline__ unsigned long long gtime() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
               : "=r"(ok) : "r"(saddr(b)), "r"(parity) : "memory");
  return ok != 0;
}
__device__ bool mbar_wait(uint64_t* b, uint32_t parity, int* err) {
  const unsigned long long t0 = gtime();
  while (!mbar_try(b, parity)) {
    if (gtime() - t0 > 1000000000ull) { *err = 1; return false; }
  }
  return true;
}

struct __align__(1024) Sm {
  unsigned char a[128 * 128];   // up to M = 128 rows x 128 bytes
  unsigned char b[256 * 128];   // up to N = 256 rows x 128 bytes
  uint64_t bar[4];
  uint32_t tmem;
};

template <int M, int N, int COLS, int MODE>
__global__ void __launch_bounds__(128) bench(int iters, long long* out, int* err) {
  extern __shared__ unsigned char raw[];
  Sm& s = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  for (int i = threadIdx.x; i < (int)(sizeof(s.a) + sizeof(s.b)) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(s.a)[i] = 0;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(&s.bar[i])));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (threadIdx.x < 32) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(&s.tmem)), "r"(COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = s.tmem;
  if (MODE == 0 ? threadIdx.x == 0 : threadIdx.x < 32) {
    const uint64_t da = desc_k(saddr(s.a)), db = desc_k(saddr(s.b));
    const uint32_t id = idesc(M, N);
    long long issue = 0;
    const long long t0 = clock64();
    bool ok = true;
    for (int it = 0; it < iters && ok; ++it) {
      if (it >= 2) ok = mbar_wait(&s.bar[it & 3 ^ 2], ((it - 2) >> 2) & 1, err);
      const long long a0 = clock64();
      if (MODE == 0) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
                       ::"r"(tmem), "l"(da + 2 * kk), "l"(db + 2 * kk), "r"(id), "r"(kk));
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(saddr(&s.bar[it & 3]))
                     : "memory");
      } else if (MODE == 1) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          asm volatile("{\n .reg .pred p, e;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
                       ::"r"(tmem), "l"(da + 2 * kk), "l"(db + 2 * kk), "r"(id), "r"(kk));
        asm volatile("{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(saddr(&s.bar[it & 3]))
                     : "memory");
      } else {
        // one asm block: elect once, four MMAs with immediate accumulate flags, commit
        asm volatile("{\n .reg .pred e, p0, p1;\n setp.ne.b32 p0, 0, 0;\n setp.eq.b32 p1, 0, 0;\n elect.sync _|e, 0xffffffff;\n"
                     " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %9, p0;\n"
                     " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %4, %9, p1;\n"
                     " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %6, %9, p1;\n"
                     " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %8, %9, p1;\n"
                     " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%10];\n}\n"
                     ::"r"(tmem), "l"(da), "l"(db), "l"(da + 2), "l"(db + 2), "l"(da + 4), "l"(db + 4), "l"(da + 6), "l"(db + 6),
                     "r"(id), "r"(saddr(&s.bar[it & 3])) : "memory");
      }
      issue += clock64() - a0;
    }
    for (int it = iters > 2 ? iters - 2 : 0; it < iters && ok; ++it) ok = mbar_wait(&s.bar[it & 3], (it >> 2) & 1, err);
    const long long t1 = clock64();
    if (threadIdx.x == 0) {
      out[blockIdx.x * 2] = t1 - t0;
      out[blockIdx.x * 2 + 1] = issue;
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (threadIdx.x < 32) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(COLS));
}

template <int M, int N, int COLS, int MODE>
void run(const char* name, int ctas_per_sm, int iters) {
  const int sms = 148, grid = sms * ctas_per_sm;
  long long* d_out;
  int* d_err;
  cudaMalloc(&d_out, grid * 2 * sizeof(long long));
  cudaMalloc(&d_err, sizeof(int));
  cudaMemset(d_err, 0, sizeof(int));
  const size_t smem = sizeof(Sm) + 1024;
  cudaFuncSetAttribute(bench<M, N, COLS, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  bench<M, N, COLS, MODE><<<grid, 128, smem>>>(2, d_out, d_err);   // warm-up
  cudaEvent_t e0, e1;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  cudaEventRecord(e0);
  bench<M, N, COLS, MODE><<<grid, 128, smem>>>(iters, d_out, d_err);
  cudaEventRecord(e1);
  cudaError_t e = cudaDeviceSynchronize();
  float ms = 0;
  cudaEventElapsedTime(&ms, e0, e1);
  long long* h = new long long[grid * 2];
  int herr = 0;
  cudaMemcpy(h, d_out, grid * 2 * sizeof(long long), cudaMemcpyDeviceToHost);
  cudaMemcpy(&herr, d_err, sizeof(int), cudaMemcpyDeviceToHost);
  double cyc = 0, iss = 0;
  for (int i = 0; i < grid; ++i) { cyc += h[2 * i]; iss += h[2 * i + 1]; }
  cyc /= grid;
  iss /= grid;
  const double mmas_per_sm = 4.0 * iters * ctas_per_sm;
  const double flops = 2.0 * M * N * 64 * iters * grid;
  printf("%-14s mode %d ctas/SM %d: %.3f ms, %.1f TFLOP/s, cycles/CTA %.0f -> %.2f cycles per MMA per SM, issue %.1f cycles per group of 4 (err %d, %s)\n",
         name, MODE, ctas_per_sm, ms, flops / (ms * 1e-3) / 1e12, cyc, cyc / mmas_per_sm, iss / iters, herr,
         cudaGetErrorString(e));
  delete[] h;
  cudaFree(d_out);
  cudaFree(d_err);
}

int main() {
  const int iters = 20000;
  for (int c : {1, 4}) {
    run<64, 64, 128, 0>("M64 N64", c, iters);
    run<64, 64, 128, 1>("M64 N64", c, iters);
    run<64, 64, 128, 2>("M64 N64", c, iters);
    run<64, 16, 128, 2>("M64 N16", c, iters);
    run<64, 32, 128, 2>("M64 N32", c, iters);
    run<64, 128, 128, 2>("M64 N128", c, iters);
    run<128, 64, 128, 0>("M128 N64", c, iters);
    run<128, 64, 128, 2>("M128 N64", c, iters);
    run<128, 128, 128, 2>("M128 N128", c, iters);
  }
  return 0;
}
