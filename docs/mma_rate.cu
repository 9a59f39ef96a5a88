// Rate of back-to-back tcgen05.mma instructions on one SM (M = 128, K = 16 per instruction,
// bf16 operands, fp32 accumulator in tensor memory): the measurement behind the backward
// kernel's design notes.  One CTA per SM, one issuing thread, KS instructions per commit, the
// commit awaited before the next batch.
//   SS: A and B K-major, 128-byte swizzled, in shared memory; TS: A in tensor memory;
//   B-MN: B MN-major (N contiguous), as the backward's dV / dK / dQ products use it.
// Build and run (one B200):
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 --expt-relaxed-constexpr \
//        -I spacetime_attention_b200/csrc -I include -o mma_rate docs/mma_rate.cu && ./mma_rate
// The operands are zeros; only the time per instruction is of interest.
#include <cstdint>
#include <cstdio>

#include <cuda_runtime.h>

#include "osp_device.cuh"

using namespace osp;

template <int N, int KS, bool kTs, bool kBmn>
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int iters, unsigned long long* cycles) {
  extern __shared__ unsigned char raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  const uint32_t base = smem_u32(sm);
  // A: 128 rows x 128 bytes (16 KB); B: up to 256 rows x 128 bytes (32 KB); then the barrier and
  // the tensor-memory address slot
  const uint32_t sA = base, sB = base + 16384, bar = base + 16384 + 32768, slot = bar + 64;
  for (int i = threadIdx.x; i < (16384 + 32768) / 16; i += blockDim.x)
    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(base + 16 * i), "r"(0u) : "memory");
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  if (threadIdx.x < 32) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + 16384 + 32768 + 64);
  const unsigned long long t0 = clock64();
  if (threadIdx.x < 32) {
    const bool leader = threadIdx.x == 0;
    constexpr uint32_t idesc = idesc_bf16_f32(128, N, kBmn);
    const uint64_t da = sdesc_sw128(sA, 16, 1024);
    const uint64_t db = kBmn ? sdesc_sw128(sB, 16384, 1024) : sdesc_sw128(sB, 16, 1024);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        // K step kk % 4 of a 64-channel K-major chunk (32 bytes each), or of 16-row MN-major groups
        const uint64_t koff = (uint64_t)(((kk & 3) * 32) >> 4);
        const uint64_t boff = kBmn ? (uint64_t)(128 * (kk & 3)) : koff;
        if constexpr (kTs) {
          if (leader) mma_ts(tmem, tmem + 256 + 8 * (kk & 3), db + boff, idesc, kk > 0 ? 1u : 0u);
        } else {
          if (leader) mma_ss(tmem, da + koff, db + boff, idesc, kk > 0 ? 1u : 0u);
        }
      }
      if (leader) tc_commit(bar);
      for (int w = 0; w < (1 << 26) && !mbar_try_wait(bar, it & 1); ++w) {
      }
    }
  }
  __syncthreads();
  const unsigned long long t1 = clock64();
  if (threadIdx.x == 0 && blockIdx.x == 0) cycles[0] = t1 - t0;
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int N, int KS, bool kTs = false, bool kBmn = false>
void run(int sms, unsigned long long* d) {
  const int iters = 2000, smem = 16384 + 32768 + 128 + 1024;
  cudaFuncSetAttribute(mma_rate_kernel<N, KS, kTs, kBmn>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  mma_rate_kernel<N, KS, kTs, kBmn><<<sms, 128, smem>>>(10, d);
  cudaDeviceSynchronize();
  mma_rate_kernel<N, KS, kTs, kBmn><<<sms, 128, smem>>>(iters, d);
  const cudaError_t e = cudaDeviceSynchronize();
  unsigned long long c = 0;
  cudaMemcpy(&c, d, 8, cudaMemcpyDeviceToHost);
  const double flop = 2.0 * 128 * N * 16 * KS * (double)iters;
  printf("%s%s N=%3d, %2d per commit: %7.1f cycles per instruction, %7.1f flop/cycle/SM (%s)\n", kTs ? "TS" : "SS",
         kBmn ? " B-MN" : "", N, KS, (double)c / (iters * KS), flop / c, cudaGetErrorString(e));
}

int main() {
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  unsigned long long* d = nullptr;
  cudaMalloc(&d, 8);
  run<64, 4>(sms, d);
  run<64, 16>(sms, d);
  run<128, 4>(sms, d);
  run<128, 16>(sms, d);
  run<256, 16>(sms, d);
  run<64, 16, true>(sms, d);
  run<128, 16, true>(sms, d);
  run<64, 16, true, true>(sms, d);
  run<64, 16, false, true>(sms, d);
  cudaFree(d);
  return 0;
}
