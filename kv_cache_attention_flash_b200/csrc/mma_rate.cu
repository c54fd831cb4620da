// Measurement program (not part of libfdllm.so): time per tcgen05.mma
// (M = 128, K = 16, bf16 operands, fp32 accumulator) issued back to back by
// one thread, for N = 16 .. 256, one, two or four accumulators, and the two
// operand layouts of the step kernel (K-major 128-byte swizzled A and B; the
// P.V form with an MN-major swizzled A and an MN-major unswizzled B). One
// CTA, zero-filled operands, every wait bounded.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdio>
#include <cstdint>
#include "ptx.cuh"

using namespace fdllm;

struct Cfg { int n; int nacc; int layout; };   // layout 0: A,B K-major SW128; 1: PV (A MN SW128, B MN noswz)

__global__ void __launch_bounds__(128, 1) bench(const Cfg* cfgs, int ncfg, int reps,
                                               unsigned long long* out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  const int tid = threadIdx.x;
  for (int i = tid; i < 65536 / 16; i += 128) reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  if (tid == 0) { ptx::mbar_init(&bar, 1); ptx::fence_mbar_init(); }
  if (tid < 32) { ptx::tmem_alloc(&tbase, 512); ptx::tmem_relinquish(); }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tbase;
  const uint32_t a0 = ptx::smem_u32(smem), b0 = ptx::smem_u32(smem + 32768);
  uint32_t phase = 0;
  for (int ci = 0; ci < ncfg; ++ci) {
    const Cfg c = cfgs[ci];
    if (tid == 0) {
      const uint32_t idesc = c.layout == 0 ? ptx::idesc_bf16_f32(128, c.n, false, false)
                                           : ptx::idesc_bf16_f32(128, c.n, true, true);
      const unsigned long long t0 = ptx::globaltimer();
      for (int r = 0; r < reps; ++r) {
        const int ks = r & 7;
        uint64_t ad, bd;
        if (c.layout == 0) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          ad = ptx::smem_desc_sw128(a0 + off, 16, 1024);
          bd = ptx::smem_desc_sw128(b0 + (ks & 3) * 32, 16, 1024);
        } else {
          ad = ptx::smem_desc_sw128(a0 + ks * 2048, 16384, 1024);
          bd = ptx::smem_desc_noswz(b0 + ks * 256, 128, 2048);
        }
        const uint32_t d = tmem + (uint32_t)((r % c.nacc) * c.n);
        ptx::umma_f16_ss(d, ad, bd, idesc, r >= c.nacc ? 1u : 0u);
      }
      const unsigned long long t1 = ptx::globaltimer();
      ptx::umma_commit(&bar);
      const bool ok = ptx::mbar_wait(&bar, phase & 1, 1000000000ull);
      const unsigned long long t2 = ptx::globaltimer();
      out[3 * ci] = t1 - t0;
      out[3 * ci + 1] = t2 - t0;
      out[3 * ci + 2] = ok;
    }
    ++phase;
    __syncthreads();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (tid < 32) ptx::tmem_dealloc(tmem, 512);
}

int main() {
  Cfg h[] = {
    {16, 1, 0}, {32, 1, 0}, {64, 1, 0}, {128, 1, 0}, {256, 1, 0},
    {32, 2, 0}, {64, 2, 0}, {128, 2, 0}, {256, 2, 0},
    {32, 4, 0}, {64, 4, 0}, {128, 4, 0},
    {32, 1, 1}, {64, 1, 1}, {128, 1, 1}, {64, 2, 1},
  };
  const int n = sizeof(h) / sizeof(h[0]);
  Cfg* d;
  unsigned long long* o;
  cudaMalloc(&d, sizeof(h));
  cudaMalloc(&o, 3 * n * sizeof(unsigned long long));
  cudaMemcpy(d, h, sizeof(h), cudaMemcpyHostToDevice);
  const int smem = 65536 + 1024;
  cudaFuncSetAttribute(bench, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const int reps = 512;
  for (int it = 0; it < 2; ++it) {
    bench<<<1, 128, smem>>>(d, n, reps, o);
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) { printf("error %s\n", cudaGetErrorString(e)); return 1; }
  }
  unsigned long long r[3 * 64];
  cudaMemcpy(r, o, 3 * n * sizeof(unsigned long long), cudaMemcpyDeviceToHost);
  for (int i = 0; i < n; ++i) {
    const double per = (double)r[3 * i + 1] / reps;
    const double flops = 2.0 * 128 * h[i].n * 16;
    printf("N=%3d acc=%d layout=%d: issue %.1f ns/mma, complete %.1f ns/mma, %.2f TFLOP/s per SM, ok=%llu\n",
           h[i].n, h[i].nacc, h[i].layout, (double)r[3 * i] / reps, per, flops / per / 1e3, r[3 * i + 2]);
  }
  return 0;
}
