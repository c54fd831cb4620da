// Output projection of the attention block: y = residual + o W_o, bf16
// operands, fp32 accumulation in TMEM (the residual added in fp32), one
// rounding to bf16.
//
// "Flash-dLLM: I/O-Aware KV Caching and Parallel Decoding for Fast,
// Memory-Efficient Diffusion LLMs" (ai4snews summary), paragraph 1, covers a
// layer up to the attention output (QKV projection, RoPE, cache write,
// scheduled attention). The projection that follows attention in a
// transformer layer is a plain GEMM over the heads' outputs side by side; it
// is read here with the conventions of Wqkv (y = x W, W row-major, no bias).
//
// One CTA per 128 x BN tile of y (BN = 256 or 128, whichever fills the SMs
// in fewer tile-times), 192 threads:
//   warp 0 (lane 0): TMA producer. Per 64-deep K step one box of o (128 rows
//     x 64 columns, K-major, 128-byte swizzle) and one box of W_o (64 K rows
//     x BN / 64 blocks of 64 columns, N-major, 128-byte swizzle), into a
//     ring of 192 KB (4 stages of 48 KB, or 6 of 32 KB).
//   warp 1 (lane 0): tcgen05.mma issuer (M128 N-BN K16, A K-major, B
//     N-major) into BN TMEM columns; owns the TMEM allocation.
//   warps 2-5: epilogue, one TMEM lane quadrant each: fp32 accumulator
//     (+ the residual row, read before the store so that y may be the
//     residual) -> bf16 (round to nearest even) -> 16-byte stores of y.
// All waits are bounded; a timeout writes FDLLM_ERR_TIMEOUT to the caller's
// status word (if given), stops the ring, drains the copies already issued
// and frees TMEM.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstddef>
#include <cstdint>

#include "fdllm.h"
#include "fdllm_internal.h"
#include "ptx.cuh"

namespace fdllm {
namespace {

constexpr int OP_BM = 128;                                // rows of y per tile (UMMA M)
constexpr int OP_BK = 64;                                 // K per stage: one 128-byte span
constexpr int OP_A_BYTES = OP_BM * OP_BK * 2;             // 16 KB
constexpr int OP_BOX_BYTES = OP_BK * 64 * 2;              // 8 KB: 64 K rows x 64 columns
constexpr int OP_PIPE_BYTES = 192 * 1024;
constexpr int OP_THREADS = 192;
constexpr int OP_MAX_STAGES = 6;
constexpr uint64_t OP_WAIT_NS = 1000000000ull;            // 1 s

// Per tile width BN (UMMA N): stage size and ring depth.
template <int BN>
struct OpCfg {
  static constexpr int B_BYTES = (BN / 64) * OP_BOX_BYTES;
  static constexpr int STAGE_BYTES = OP_A_BYTES + B_BYTES;      // 48 KB or 32 KB
  static constexpr int STAGES = OP_PIPE_BYTES / STAGE_BYTES;    // 4 or 6
  static_assert(STAGES <= OP_MAX_STAGES && STAGES * STAGE_BYTES == OP_PIPE_BYTES, "ring");
};

struct OpCtrl {
  uint64_t full[OP_MAX_STAGES];
  uint64_t empty[OP_MAX_STAGES];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

constexpr int OP_SMEM_BYTES = OP_PIPE_BYTES + 1024 + 1024;   // ring, control, alignment slack
static_assert(sizeof(OpCtrl) <= 1024, "control block");

__device__ __forceinline__ bool op_wait(OpCtrl* c, uint64_t* bar, uint32_t parity,
                                        int32_t* status) {
  if (*reinterpret_cast<volatile int*>(&c->abort)) return false;
  if (ptx::mbar_wait(bar, parity, OP_WAIT_NS)) return true;
  atomicExch(&c->abort, 1);
  if (status) atomicExch(reinterpret_cast<int*>(status), (int)FDLLM_ERR_TIMEOUT);
  return false;
}

template <int BN>
__global__ void __launch_bounds__(OP_THREADS, 1)
    oproj_kernel(const __grid_constant__ CUtensorMap tmap_o, const __grid_constant__ CUtensorMap tmap_w,
                 const __nv_bfloat16* resid, __nv_bfloat16* y, int rows, int hidden,
                 int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  OpCtrl* ctrl = reinterpret_cast<OpCtrl*>(smem + OP_PIPE_BYTES);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int m0 = blockIdx.x * OP_BM;
  constexpr int STAGES = OpCfg<BN>::STAGES;
  constexpr int STAGE_BYTES = OpCfg<BN>::STAGE_BYTES;
  const int n0 = blockIdx.y * BN;
  const int nkb = hidden / OP_BK;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&ctrl->full[s], 1);
      ptx::mbar_init(&ctrl->empty[s], 1);
    }
    ptx::mbar_init(&ctrl->done, 1);
    ctrl->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&ctrl->tmem_base, BN);
    ptx::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmap_o);
    ptx::prefetch_tmap(&tmap_w);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES;
        const uint32_t u = kb / STAGES;
        if (u > 0 && !op_wait(ctrl, &ctrl->empty[s], (u - 1) & 1, status)) break;
        uint8_t* st = smem + s * STAGE_BYTES;
        ptx::mbar_arrive_expect_tx(&ctrl->full[s], STAGE_BYTES);
        ptx::tma_load_2d(st, &tmap_o, kb * OP_BK, m0, &ctrl->full[s]);
        ptx::tma_load_3d(st + OP_A_BYTES, &tmap_w, 0, kb * OP_BK, n0 / 64, &ctrl->full[s]);
        ++issued;
      }
      // the copies this thread issued have landed before the CTA exits
      // (they have, unless a wait timed out)
      for (int kb = issued > STAGES ? issued - STAGES : 0; kb < issued; ++kb)
        ptx::mbar_wait(&ctrl->full[kb % STAGES], (kb / STAGES) & 1, OP_WAIT_NS);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(OP_BM, BN, false, true);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES;
        const uint32_t u = kb / STAGES;
        if (!op_wait(ctrl, &ctrl->full[s], u & 1, status)) break;
        ptx::tc_fence_after();
        const uint32_t a_base = ptx::smem_u32(smem + s * STAGE_BYTES);
        const uint32_t b_base = a_base + OP_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < OP_BK / 16; ++kk) {
          // A: K-major rows of 128 bytes, 8-row atoms 1024 bytes apart.
          const uint64_t ad = ptx::smem_desc_sw128(a_base + kk * 32, 16, 1024);
          // B: N-major; the 64-column boxes 8 KB apart, 8-row K groups
          // 1024 bytes apart; a K16 slice is 16 rows = 2 KB.
          const uint64_t bd = ptx::smem_desc_sw128(b_base + kk * 2048, OP_BOX_BYTES, 1024);
          ptx::umma_f16_ss(tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        ptx::umma_commit(&ctrl->empty[s]);
      }
      ptx::umma_commit(&ctrl->done);
      // every MMA of this thread has completed before TMEM is freed
      ptx::mbar_wait(&ctrl->done, 0, OP_WAIT_NS);
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32 * (w % 4) .. + 31 (rows of the tile)
    const int quad = warp & 3;
    const int row = m0 + quad * 32 + lane;
    const bool ok = __all_sync(0xffffffffu, op_wait(ctrl, &ctrl->done, 0, status));
    ptx::tc_fence_after();
    if (ok) {
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16);
      __nv_bfloat16* yrow = y + (size_t)row * hidden + n0;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        float v[32];
        ptx::tmem_ld32(taddr + c0, v);
        ptx::tmem_ld_wait();
        if (row < rows) {
          if (resid) {   // read before the store: y may be the residual itself
            const uint4* rsrc =
                reinterpret_cast<const uint4*>(resid + (size_t)row * hidden + n0 + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 r4 = rsrc[q];
              const uint32_t rw[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                v[8 * q + 2 * e] += __uint_as_float(rw[e] << 16);
                v[8 * q + 2 * e + 1] += __uint_as_float(rw[e] & 0xffff0000u);
              }
            }
          }
          uint4* dst = reinterpret_cast<uint4*>(yrow + c0);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(ptx::pack_bf16(v[8 * q], v[8 * q + 1]),
                                ptx::pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                                ptx::pack_bf16(v[8 * q + 4], v[8 * q + 5]),
                                ptx::pack_bf16(v[8 * q + 6], v[8 * q + 7]));
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) ptx::tmem_dealloc(tmem, BN);
}

template <int BN>
cudaError_t launch_oproj_bn(const void* tmap_o, const void* tmap_w, const void* resid, void* y,
                            int rows, int hidden, int32_t* status, cudaStream_t stream) {
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = opt_in_smem(reinterpret_cast<const void*>(oproj_kernel<BN>), OP_SMEM_BYTES,
                              attr_done);
  if (e != cudaSuccess) return e;
  dim3 grid((rows + OP_BM - 1) / OP_BM, hidden / BN);
  oproj_kernel<BN><<<grid, OP_THREADS, OP_SMEM_BYTES, stream>>>(
      *reinterpret_cast<const CUtensorMap*>(tmap_o), *reinterpret_cast<const CUtensorMap*>(tmap_w),
      reinterpret_cast<const __nv_bfloat16*>(resid), reinterpret_cast<__nv_bfloat16*>(y), rows,
      hidden, status);
  return cudaGetLastError();
}

}  // namespace

size_t oproj_smem_bytes() { return OP_SMEM_BYTES; }

cudaError_t launch_oproj(const void* tmap_o, const void* tmap_w, int bn, const void* resid,
                         void* y, int rows, int hidden, int32_t* status, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  if (bn == 256)
    return launch_oproj_bn<256>(tmap_o, tmap_w, resid, y, rows, hidden, status, stream);
  if (bn == 128)
    return launch_oproj_bn<128>(tmap_o, tmap_w, resid, y, rows, hidden, status, stream);
  return cudaErrorInvalidValue;
}

}  // namespace fdllm
