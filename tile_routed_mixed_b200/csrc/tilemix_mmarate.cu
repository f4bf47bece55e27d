// Tensor-core rate of the MMA forms the fused prefill kernel issues, measured
// on the device: one thread per CTA issues back-to-back tcgen05.mma of one
// kind and shape into TMEM, timed on the SM clock.  A measurement of the
// hardware for the mixed roofline's INT8 : FP16 rate ratio, not a step of the
// attention method.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tilemix.h"
#include "tilemix_internal.h"
#include "tilemix_ptx.cuh"

namespace tilemix {
namespace {

constexpr int kRateThreads = 128;
constexpr int kRateSmem = 16384 + 32768 + 1024;  // A tile, B tile, alignment slack

// Forms: 0 kind::f16 with A and B in shared memory (the FP16 score tiles),
// 1 kind::i8 likewise (the INT8 score tiles), 2 kind::f16 with A in TMEM and
// B MN-major (P.V), 3 kind::f8f6f4 e4m3 in shared memory (the FP8 score tiles).
template <int kForm, int N>
__global__ void __launch_bounds__(kRateThreads, 1)
    mma_rate_kernel(int iters, unsigned long long timeout_ns, long long* out) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  // operands: small nonzero values (every byte pattern is a finite fp16,
  // int8 or e4m3 code of small magnitude)
  for (int i = threadIdx.x; i < (16384 + 32768) / 4; i += kRateThreads)
    reinterpret_cast<uint32_t*>(sm)[i] = 0x11213141u ^ (static_cast<uint32_t>(i) * 0x01000101u & 0x0f0f0f0fu);
  if (threadIdx.x < 32) {
    ptx::tmem_alloc(&tmem_base, 512);
    ptx::tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base;
  if (threadIdx.x == 0) {
    const uint32_t a = ptx::smem_addr(sm), b = a + 16384;
    const uint64_t tk = ptx::smem_desc(0, 16, 1024, ptx::kSwizzle128B);   // K-major
    const uint64_t tmn = ptx::smem_desc(0, 8192, 1024, ptx::kSwizzle128B);  // MN-major, 64-col chunks 8 KB apart
    const auto at = [](uint64_t t, uint32_t addr) {
      return t | static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    };
    const long long t0 = clock64();
    for (int i = 0; i < iters; ++i) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t acc = (i > 0 || k > 0) ? 1u : 0u;
        if constexpr (kForm == 0)
          ptx::mma_f16_ss(tmem, at(tk, a + k * 32), at(tk, b + k * 32), ptx::idesc_f16(128, N, false), acc);
        else if constexpr (kForm == 1)
          ptx::mma_i8_ss(tmem, at(tk, a + k * 32), at(tk, b + k * 32), ptx::idesc_s8(128, N), acc);
        else if constexpr (kForm == 2)
          ptx::mma_f16_ts(tmem, tmem + 256 + k * 8, at(tmn, b + k * 2048), ptx::idesc_f16(128, N, true), acc);
        else
          ptx::mma_f8_ss(tmem, at(tk, a + k * 32), at(tk, b + k * 32), ptx::idesc_f16(128, N, false), acc);
      }
    }
    const long long t1 = clock64();
    ptx::mma_commit(&bar);
    const unsigned long long start = ptx::globaltimer();
    bool done = true;
    while (!ptx::mbar_try_wait(&bar, 0)) {
      if (ptx::globaltimer() - start > timeout_ns) {  // reported as -1
        done = false;
        break;
      }
    }
    const long long t2 = clock64();
    out[2 * blockIdx.x] = t1 - t0;
    out[2 * blockIdx.x + 1] = done ? t2 - t0 : -1;
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

template <int kForm, int N>
int launch_rate(int iters, int ctas, long long* out, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(mma_rate_kernel<kForm, N>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kRateSmem);
  if (e != cudaSuccess) return static_cast<int>(e);
  mma_rate_kernel<kForm, N><<<ctas, kRateThreads, kRateSmem, st>>>(iters, 2000000000ull, out);
  return static_cast<int>(cudaGetLastError());
}

template <int kForm>
int launch_rate_n(int n, int iters, int ctas, long long* out, cudaStream_t st) {
  if (n == 64) return launch_rate<kForm, 64>(iters, ctas, out, st);
  if (n == 128) return launch_rate<kForm, 128>(iters, ctas, out, st);
  return launch_rate<kForm, 256>(iters, ctas, out, st);
}

}  // namespace
}  // namespace tilemix

extern "C" TILEMIX_API int tilemix_mma_rate(int form, int n, int iters, int ctas,
                                            long long* cycles_dev, void* stream) {
  if (form < 0 || form > 3 || (n != 64 && n != 128 && n != 256) || iters < 1 ||
      iters > (1 << 20) || ctas < 1 || ctas > 4096 || !cycles_dev)
    return TILEMIX_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc;
  switch (form) {
    case 0: rc = tilemix::launch_rate_n<0>(n, iters, ctas, cycles_dev, st); break;
    case 1: rc = tilemix::launch_rate_n<1>(n, iters, ctas, cycles_dev, st); break;
    case 2: rc = tilemix::launch_rate_n<2>(n, iters, ctas, cycles_dev, st); break;
    default: rc = tilemix::launch_rate_n<3>(n, iters, ctas, cycles_dev, st); break;
  }
  return rc == cudaSuccess ? TILEMIX_OK : TILEMIX_ERR_CUDA;
}
