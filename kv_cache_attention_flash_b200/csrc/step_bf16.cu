// Flash-Cache fused layer step for bf16 on sm_100a.
//
// One CTA per (row group g, head h). A row group packs whole sequences into
// at most 128 query rows, so every fresh key/value a sequence attends to is
// produced by the CTA that attends to it, and no grid-wide ordering is
// needed ("Flash-dLLM: I/O-Aware KV Caching and Parallel Decoding for Fast,
// Memory-Efficient Diffusion LLMs", ai4snews summary, paragraph 1: QKV
// projection, RoPE and the cache write fused, K/V written to the cache from
// on-chip memory; scheduled attention aligns each query block with its own
// KV blocks through a block table).
//
// Phase 1 (projection, tensor cores): [128 rows x H] x [H x 384] where the
//   384 columns are this head's q | k | v blocks of Wqkv. TMA streams x and
//   Wqkv tiles (128-byte swizzle) through a 3-stage mbarrier pipeline; one
//   thread issues tcgen05.mma (M=128, N=128, K=16, bf16 -> fp32) into a
//   512-column TMEM accumulator.
// Phase 2 (epilogue): all 8 warps read TMEM (warp w owns lanes 32*(w%4)..),
//   apply rotate-half RoPE to q and k from an fp32 cos/sin table, round to
//   bf16, keep q in shared memory and stage k/v rows, which are then copied
//   to their cache slots with coalesced 16-byte stores.
// Phase 3 (attention): per sequence of the group, two passes over the
//   sequence's keys (the context slots [0, L_b) through the block table, then
//   the view rows' fresh slots), 64 keys per chunk staged by cp.async:
//   pass 1 finds each row's log-sum-exp, pass 2 forms the exact
//   probabilities, accumulates P.V and the per-key column sums of P (the
//   attention mass), with mma.sync m16n8k16 on bf16 operands.
//   The Flash-Verify two-view rule (paragraph 3 of the same page) decides
//   visibility of the fresh view keys.
#include <cuda.h>
#include <cuda_bf16.h>

#include "fdllm_internal.h"
#include "ptx.cuh"

namespace fdllm {
namespace {

constexpr int D = 128;            // head_dim served by this kernel
constexpr int BM = 128;           // rows per group (UMMA M)
constexpr int BK = 64;            // K per pipeline stage (one 128-byte swizzle span)
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;           // 16 KB
constexpr int BOX_BYTES = BK * 64 * 2;         // 8 KB: 64 K-rows x 64 columns
constexpr int B_BYTES = 6 * BOX_BYTES;         // q, k, v blocks, two boxes each
constexpr int STAGE_BYTES = A_BYTES + B_BYTES; // 64 KB
constexpr int PIPE_BYTES = STAGES * STAGE_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int NTHREADS = 256;
constexpr int KC = 64;                          // keys per attention chunk
constexpr uint64_t WAIT_NS = 1000000000ull;     // bounded waits: 1 s

// Reuse of the pipeline area after the projection.
constexpr int Q_OFF = 0;                  // q tile, bf16 [128][128], 16-byte chunks swizzled
constexpr int KST_OFF = 32768;            // fresh k rows (staging)
constexpr int VST_OFF = 65536;            // fresh v rows (staging)
constexpr int KV_OFF = 98304;             // 2 x (K chunk 16 KB + V chunk 16 KB)
constexpr int KV_BUF = 2 * KC * D * 2;    // 32 KB per buffer
constexpr int OBUF_OFF = 32768;           // O partials (after staging/KV are idle)
constexpr int OBUF_LD = 136;              // padded row length (floats)
constexpr int MISC_OFF = KV_OFF + 2 * KV_BUF;   // 163840
constexpr int LSE_OFF = MISC_OFF;               // float[128]
constexpr int STAT_OFF = LSE_OFF + 512;         // float2[8 warps][16 rows]
constexpr int MASSB_OFF = STAT_OFF + 1024;      // float[8][64]
constexpr int XROW_OFF = MASSB_OFF + 2048;      // int[128] view rows of the sequence
static_assert(XROW_OFF + 512 + 64 <= PIPE_BYTES, "misc area overflows");
static_assert(OBUF_OFF + 8 * 16 * OBUF_LD * 4 <= MISC_OFF, "O buffer overflows");

struct Ctrl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int nx;                 // view rows of the current sequence
  int row_pos[BM];
  int row_slot[BM];
  int row_page[BM];       // -1: row has bad metadata
  int row_view[BM];
};
constexpr int CTRL_OFF = PIPE_BYTES;
constexpr int SMEM_BYTES = PIPE_BYTES + (int)sizeof(Ctrl) + 1024;

__device__ __forceinline__ void set_err(int* err, int code, int detail) {
  if (atomicCAS(err, 0, code) == 0) err[1] = detail;
}

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * 256 + ((chunk ^ (row & 7)) << 4));
}

// TMEM -> registers -> RoPE -> bf16 -> swizzled shared rows. Every lane of
// the warp executes the TMEM loads; only valid rows are rotated/written.
__device__ __forceinline__ void epi_rope(uint32_t taddr, int row, bool valid, int pos,
                                         const float* cos_t, const float* sin_t, uint8_t* dst) {
#pragma unroll 1
  for (int c = 0; c < 2; ++c) {
    float lo[32], hi[32];
    ptx::tmem_ld32(taddr + 32 * c, lo);
    ptx::tmem_ld32(taddr + 64 + 32 * c, hi);
    ptx::tmem_ld_wait();
    if (!valid) {
#pragma unroll
      for (int t = 0; t < 32; ++t) lo[t] = hi[t] = 0.f;
    } else {
      const float4* cp = reinterpret_cast<const float4*>(cos_t + (size_t)pos * (D / 2) + 32 * c);
      const float4* sp = reinterpret_cast<const float4*>(sin_t + (size_t)pos * (D / 2) + 32 * c);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float4 cs = __ldg(cp + u), sn = __ldg(sp + u);
        float cv[4] = {cs.x, cs.y, cs.z, cs.w}, sv[4] = {sn.x, sn.y, sn.z, sn.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = 4 * u + e;
          const float a = lo[t], b = hi[t];
          lo[t] = a * cv[e] - b * sv[e];
          hi[t] = b * cv[e] + a * sv[e];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint4 vl, vh;
      vl.x = ptx::pack_bf16(lo[8 * u + 0], lo[8 * u + 1]);
      vl.y = ptx::pack_bf16(lo[8 * u + 2], lo[8 * u + 3]);
      vl.z = ptx::pack_bf16(lo[8 * u + 4], lo[8 * u + 5]);
      vl.w = ptx::pack_bf16(lo[8 * u + 6], lo[8 * u + 7]);
      vh.x = ptx::pack_bf16(hi[8 * u + 0], hi[8 * u + 1]);
      vh.y = ptx::pack_bf16(hi[8 * u + 2], hi[8 * u + 3]);
      vh.z = ptx::pack_bf16(hi[8 * u + 4], hi[8 * u + 5]);
      vh.w = ptx::pack_bf16(hi[8 * u + 6], hi[8 * u + 7]);
      *reinterpret_cast<uint4*>(dst + swz(row, 4 * c + u)) = vl;
      *reinterpret_cast<uint4*>(dst + swz(row, 8 + 4 * c + u)) = vh;
    }
  }
}

__device__ __forceinline__ void epi_plain(uint32_t taddr, int row, bool valid, uint8_t* dst) {
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    float v[32];
    ptx::tmem_ld32(taddr + 32 * c, v);
    ptx::tmem_ld_wait();
    if (!valid) {
#pragma unroll
      for (int t = 0; t < 32; ++t) v[t] = 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint4 w;
      w.x = ptx::pack_bf16(v[8 * u + 0], v[8 * u + 1]);
      w.y = ptx::pack_bf16(v[8 * u + 2], v[8 * u + 3]);
      w.z = ptx::pack_bf16(v[8 * u + 4], v[8 * u + 5]);
      w.w = ptx::pack_bf16(v[8 * u + 6], v[8 * u + 7]);
      *reinterpret_cast<uint4*>(dst + swz(row, 4 * c + u)) = w;
    }
  }
}

__global__ void __launch_bounds__(NTHREADS, 1)
    step_bf16_kernel(const __grid_constant__ StepPlan plan, const __grid_constant__ StepArgs a,
                     const __grid_constant__ CUtensorMap tmap_x,
                     const __grid_constant__ CUtensorMap tmap_w) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + CTRL_OFF);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int h = blockIdx.x / plan.n_groups;
  const int g = blockIdx.x % plan.n_groups;
  const int row0 = plan.group_row0[g];
  const int nrows = plan.group_row0[g + 1] - row0;
  const int seq_a = plan.group_seq0[g];
  const int seq_b = plan.group_seq0[g + 1];
  const int H = a.hidden;
  const int nkb = H / BK;
  const int ps = a.page_size;
  const int layer = plan.layer;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&ctrl->full[s], 1);
      ptx::mbar_init(&ctrl->empty[s], 1);
    }
    ptx::mbar_init(&ctrl->mma_done, 1);
    ctrl->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&ctrl->tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (tid == 32 * 2) {
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_w);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES;
        const int u = kb / STAGES;
        if (u > 0 && !ptx::mbar_wait(&ctrl->empty[s], (u - 1) & 1, WAIT_NS)) {
          set_err(a.err, kDevTimeout, 1);
          atomicExch(&ctrl->abort, 1);
          break;
        }
        uint8_t* st = smem + s * STAGE_BYTES;
        ptx::mbar_arrive_expect_tx(&ctrl->full[s], STAGE_BYTES);
        ptx::tma_load_2d(st, &tmap_x, kb * BK, row0, &ctrl->full[s]);
#pragma unroll
        for (int blk = 0; blk < 3; ++blk)
#pragma unroll
          for (int half = 0; half < 2; ++half)
            ptx::tma_load_2d(st + A_BYTES + (blk * 2 + half) * BOX_BYTES, &tmap_w,
                             blk * H + h * D + half * 64, kb * BK, &ctrl->full[s]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(BM, 128, false, true);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES;
        const int u = kb / STAGES;
        if (!ptx::mbar_wait(&ctrl->full[s], u & 1, WAIT_NS)) {
          set_err(a.err, kDevTimeout, 2);
          atomicExch(&ctrl->abort, 1);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a_base = ptx::smem_u32(smem + s * STAGE_BYTES);
        const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          // A: K-major rows of 128 bytes; 8-row atoms 1024 bytes apart.
          const uint64_t ad = ptx::smem_desc_sw128(a_base + kk * 32, 16, 1024);
#pragma unroll
          for (int blk = 0; blk < 3; ++blk) {
            // B: N-major (Wqkv rows are K); 64-column boxes 8 KB apart,
            // 8-row K groups 1024 bytes apart; K16 slice = 16 rows = 2 KB.
            const uint64_t bd = ptx::smem_desc_sw128(b_base + blk * 2 * BOX_BYTES + kk * 2048,
                                                     BOX_BYTES, 1024);
            ptx::umma_f16_ss(tmem + blk * 128, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
        }
        ptx::umma_commit(&ctrl->empty[s]);
      }
      ptx::umma_commit(&ctrl->mma_done);
    }
  } else {
    // ------------------------------------------------ row metadata (warps 2..7)
    for (int i = tid - 64; i < BM; i += NTHREADS - 64) {
      int pos = 0, slot = 0, page = -1, view = 0;
      if (i < nrows) {
        const int gr = row0 + i;
        pos = a.positions[gr];
        slot = a.slots ? a.slots[gr] : pos;
        view = a.view ? (int)a.view[gr] : 0;
        int b = seq_a;
        while (b + 1 < seq_b && plan.cu_rows[b + 1] <= gr) ++b;
        if (pos < 0 || pos >= a.max_position) {
          set_err(a.err, kDevBadPosition, gr);
        } else if (slot < 0 || slot >= plan.row_stride) {
          set_err(a.err, kDevBadSlot, gr);
        } else {
          const int pg = a.block_table[(size_t)b * plan.max_blocks + slot / ps];
          if (pg < 0 || pg >= a.num_pages)
            set_err(a.err, kDevBadPage, gr);
          else
            page = pg;
        }
      }
      ctrl->row_pos[i] = pos;
      ctrl->row_slot[i] = slot;
      ctrl->row_page[i] = page;
      ctrl->row_view[i] = view;
    }
  }
  __syncwarp();
  __syncthreads();   // row metadata visible; producer/MMA loops issued

  // ------------------------------------------------------------ epilogue
  const bool acc_ok = ptx::mbar_wait(&ctrl->mma_done, 0, WAIT_NS);
  if (!acc_ok) set_err(a.err, kDevTimeout, 3);
  __syncwarp();
  ptx::tc_fence_after();
  {
    const int quad = warp & 3;
    const int i = quad * 32 + lane;
    const bool valid = acc_ok && i < nrows && ctrl->row_page[i] >= 0;
    const int pos = ctrl->row_pos[i];
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    if (warp < 4) {
      epi_rope(trow + 0, i, valid, pos, a.rope_cos, a.rope_sin, smem + Q_OFF);
    } else {
      epi_rope(trow + 128, i, valid, pos, a.rope_cos, a.rope_sin, smem + KST_OFF);
      epi_plain(trow + 256, i, valid, smem + VST_OFF);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) ptx::tmem_dealloc(tmem, TMEM_COLS);

  // Fresh k/v rows -> cache slots (16 consecutive threads per 256-byte row).
  {
    const size_t head_stride = (size_t)ps * D;
    __nv_bfloat16* kp = reinterpret_cast<__nv_bfloat16*>(a.k_pool);
    __nv_bfloat16* vp = reinterpret_cast<__nv_bfloat16*>(a.v_pool);
    for (int idx = tid; idx < nrows * 32; idx += NTHREADS) {
      const int r = idx >> 5;
      const int part = idx & 31;
      const int ch = part & 15;
      const int page = ctrl->row_page[r];
      if (page < 0) continue;
      const int slot = ctrl->row_slot[r];
      const size_t off = (((size_t)layer * a.num_pages + page) * a.n_heads + h) * head_stride +
                         (size_t)(slot % ps) * D + ch * 8;
      const uint8_t* src = smem + (part < 16 ? KST_OFF : VST_OFF) + swz(r, ch);
      __nv_bfloat16* dst = (part < 16 ? kp : vp) + off;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    }
  }
  __syncthreads();   // cache writes of this CTA visible to its own threads

  // ------------------------------------------------------------ attention
  const float sl2 = 1.4426950408889634f * rsqrtf((float)D);   // log2(e) / sqrt(D)
  const uint8_t* qs = smem + Q_OFF;
  float* lse = reinterpret_cast<float*>(smem + LSE_OFF);
  float2* stat = reinterpret_cast<float2*>(smem + STAT_OFF);
  float* massb = reinterpret_cast<float*>(smem + MASSB_OFF);
  int* xrow = reinterpret_cast<int*>(smem + XROW_OFF);
  const __nv_bfloat16* kpool = reinterpret_cast<const __nv_bfloat16*>(a.k_pool);
  const __nv_bfloat16* vpool = reinterpret_cast<const __nv_bfloat16*>(a.v_pool);
  const size_t layer_base = (size_t)layer * a.num_pages * a.n_heads * ps * D;
  const int qd = lane & 3;     // quad lane: column pair
  const int gq = lane >> 2;    // row within the 8-row half

  for (int b = seq_a; b < seq_b; ++b) {
    const int ra = plan.cu_rows[b] - row0;
    const int n = plan.cu_rows[b + 1] - plan.cu_rows[b];
    if (n == 0) continue;
    const int L = plan.seq_lens[b];
    if (tid == 0) {
      int nx = 0;
      for (int r = 0; r < n; ++r)
        if (ctrl->row_view[ra + r] != 0) xrow[nx++] = ra + r;
      ctrl->nx = nx;
    }
    __syncthreads();
    const int nx = ctrl->nx;
    const int nk = L + nx;
    const int nchunks = (nk + KC - 1) / KC;
    const int n_mt = (n + 15) >> 4;
    int n_split = 8 / n_mt;
    if (n_split > 4) n_split = 4;
    if (n_split < 1) n_split = 1;
    const int KW = KC / n_split;          // 16, 32 or 64 keys per warp per chunk
    const int mt = warp % n_mt;
    const int sp = warp / n_mt;
    const bool active = sp < n_split;
    const int r_lo = 16 * mt + gq;        // sequence-local rows of this thread
    const int r_hi = r_lo + 8;
    const bool v_lo = r_lo < n, v_hi = r_hi < n;
    const int view_lo = v_lo ? ctrl->row_view[ra + r_lo] : 0;
    const int view_hi = v_hi ? ctrl->row_view[ra + r_hi] : 0;
    const int pos_lo = v_lo ? ctrl->row_pos[ra + r_lo] : 0;
    const int pos_hi = v_hi ? ctrl->row_pos[ra + r_hi] : 0;
    const int* bt = a.block_table + (size_t)b * plan.max_blocks;
    float* part = a.mass_part ? a.mass_part + ((size_t)h * plan.batch + b) * plan.row_stride
                              : nullptr;

    // Chunk loader: keys [KC*c, KC*c + KC) of this sequence, K (and V).
    auto load_chunk = [&](int c, int buf, bool with_v) {
      uint8_t* kd = smem + KV_OFF + buf * KV_BUF;
      uint8_t* vd = kd + KC * D * 2;
      for (int pi = tid; pi < KC * 16; pi += NTHREADS) {
        const int kr = pi >> 4;
        const int ch = pi & 15;
        const int j = c * KC + kr;
        const void* ksrc = kpool;
        const void* vsrc = vpool;
        uint32_t bytes = 0;
        if (j < nk) {
          int slot, page;
          if (j < L) {
            slot = j;
            page = bt[j / ps];
            if (page < 0 || page >= a.num_pages) {
              set_err(a.err, kDevBadPage, -1 - j);
              page = -1;
            }
          } else {
            const int xr = xrow[j - L];
            slot = ctrl->row_slot[xr];
            page = ctrl->row_page[xr];
          }
          if (page >= 0) {
            const size_t off = layer_base + ((size_t)page * a.n_heads + h) * ps * D +
                               (size_t)(slot % ps) * D + ch * 8;
            ksrc = kpool + off;
            vsrc = vpool + off;
            bytes = 16;
          }
        }
        ptx::cp_async16(kd + swz(kr, ch), ksrc, bytes);
        if (with_v) ptx::cp_async16(vd + swz(kr, ch), vsrc, bytes);
      }
      ptx::cp_async_commit();
    };

    // Visibility of chunk-local key kj (global key index j) for a row.
    auto visible = [&](int j, int rview, int rpos) -> bool {
      if (j >= nk) return false;
      if (j < L) return true;
      if (rview == 0) return false;
      const int xr = xrow[j - L];
      return ctrl->row_view[xr] == rview && ctrl->row_pos[xr] <= rpos;
    };

    // S = q k^T for this warp's 16 rows x KW keys of the chunk in `buf`.
    auto compute_s = [&](int buf, float (*sacc)[4]) {
      const uint8_t* kd = smem + KV_OFF + buf * KV_BUF;
      const int nt = KW / 8;
#pragma unroll
      for (int t = 0; t < 8; ++t)
        sacc[t][0] = sacc[t][1] = sacc[t][2] = sacc[t][3] = 0.f;
      int qrow = ra + 16 * mt + (lane & 15);
      if (qrow > BM - 1) qrow = BM - 1;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t af[4];
        ptx::ldmatrix_x4(af, qs + swz(qrow, 2 * kk + (lane >> 4)));
#pragma unroll
        for (int t2 = 0; t2 < 4; ++t2) {
          if (2 * t2 < nt) {
            const int krow = sp * KW + 16 * t2 + (lane & 7) + ((lane >> 4) << 3);
            uint32_t bf[4];
            ptx::ldmatrix_x4(bf, kd + swz(krow, 2 * kk + ((lane >> 3) & 1)));
            ptx::mma_bf16_16816(sacc[2 * t2], af, bf);
            ptx::mma_bf16_16816(sacc[2 * t2 + 1], af, bf + 2);
          }
        }
      }
    };

    // -------------------------------------------- pass 1: row log-sum-exp
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
    load_chunk(0, 0, false);
    for (int c = 0; c < nchunks; ++c) {
      if (c + 1 < nchunks) {
        load_chunk(c + 1, (c + 1) & 1, false);
        ptx::cp_async_wait<1>();
      } else {
        ptx::cp_async_wait<0>();
      }
      __syncthreads();
      if (active) {
        float sacc[8][4];
        compute_s(c & 1, sacc);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (t < KW / 8) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int j = c * KC + sp * KW + 8 * t + 2 * qd + e;
              if (v_lo && visible(j, view_lo, pos_lo)) {
                const float x = sacc[t][e] * sl2;
                if (x > m_lo) {
                  l_lo = l_lo * exp2f(m_lo - x) + 1.f;
                  m_lo = x;
                } else {
                  l_lo += exp2f(x - m_lo);
                }
              }
              if (v_hi && visible(j, view_hi, pos_hi)) {
                const float x = sacc[t][2 + e] * sl2;
                if (x > m_hi) {
                  l_hi = l_hi * exp2f(m_hi - x) + 1.f;
                  m_hi = x;
                } else {
                  l_hi += exp2f(x - m_hi);
                }
              }
            }
          }
        }
      }
      __syncthreads();
    }
    // combine over the 4 lanes of a quad, then over the key splits
    if (active) {
#pragma unroll
      for (int off = 1; off <= 2; off <<= 1) {
        const float mo_lo = __shfl_xor_sync(0xffffffffu, m_lo, off);
        const float lo_lo = __shfl_xor_sync(0xffffffffu, l_lo, off);
        const float mo_hi = __shfl_xor_sync(0xffffffffu, m_hi, off);
        const float lo_hi = __shfl_xor_sync(0xffffffffu, l_hi, off);
        float mn = fmaxf(m_lo, mo_lo);
        l_lo = (mn == -INFINITY) ? 0.f : l_lo * exp2f(m_lo - mn) + lo_lo * exp2f(mo_lo - mn);
        m_lo = mn;
        mn = fmaxf(m_hi, mo_hi);
        l_hi = (mn == -INFINITY) ? 0.f : l_hi * exp2f(m_hi - mn) + lo_hi * exp2f(mo_hi - mn);
        m_hi = mn;
      }
      if (qd == 0) {
        stat[warp * 16 + gq] = make_float2(m_lo, l_lo);
        stat[warp * 16 + gq + 8] = make_float2(m_hi, l_hi);
      }
    }
    __syncthreads();
    if (tid < n_mt * 16) {
      const int mt2 = tid >> 4, rr = tid & 15;
      float M = -INFINITY;
      for (int s2 = 0; s2 < n_split; ++s2) M = fmaxf(M, stat[(s2 * n_mt + mt2) * 16 + rr].x);
      float Ls = 0.f;
      if (M != -INFINITY)
        for (int s2 = 0; s2 < n_split; ++s2) {
          const float2 st = stat[(s2 * n_mt + mt2) * 16 + rr];
          Ls += st.y * exp2f(st.x - M);
        }
      lse[tid] = (Ls > 0.f) ? M + log2f(Ls) : INFINITY;
    }
    // zero this head's mass row past the context; view slots are filled below
    if (part)
      for (int j = L + tid; j < plan.row_stride; j += NTHREADS) part[j] = 0.f;
    __syncthreads();

    // -------------------------------------------- pass 2: P, P.V, mass
    const float lse_lo = lse[16 * mt + gq];
    const float lse_hi = lse[16 * mt + gq + 8];
    float oacc[16][4];
#pragma unroll
    for (int t = 0; t < 16; ++t) oacc[t][0] = oacc[t][1] = oacc[t][2] = oacc[t][3] = 0.f;
    load_chunk(0, 0, true);
    for (int c = 0; c < nchunks; ++c) {
      if (c + 1 < nchunks) {
        load_chunk(c + 1, (c + 1) & 1, true);
        ptx::cp_async_wait<1>();
      } else {
        ptx::cp_async_wait<0>();
      }
      __syncthreads();
      if (active) {
        float sacc[8][4];
        compute_s(c & 1, sacc);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (t < KW / 8) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int j = c * KC + sp * KW + 8 * t + 2 * qd + e;
              const float p_lo = (v_lo && visible(j, view_lo, pos_lo))
                                     ? exp2f(sacc[t][e] * sl2 - lse_lo) : 0.f;
              const float p_hi = (v_hi && visible(j, view_hi, pos_hi))
                                     ? exp2f(sacc[t][2 + e] * sl2 - lse_hi) : 0.f;
              sacc[t][e] = p_lo;
              sacc[t][2 + e] = p_hi;
              // column sums over the warp's 16 rows
              float cs = p_lo + p_hi;
              cs += __shfl_xor_sync(0xffffffffu, cs, 4);
              cs += __shfl_xor_sync(0xffffffffu, cs, 8);
              cs += __shfl_xor_sync(0xffffffffu, cs, 16);
              if (gq == 0) massb[mt * KC + sp * KW + 8 * t + 2 * qd + e] = cs;
            }
          }
        }
        // O += P V over the warp's KW keys, 16 keys per MMA step. P enters
        // the tensor cores as bf16 hi + lo parts (P - hi rounded again), so
        // the product carries ~16 significant bits of P; V is exact bf16.
        const uint8_t* vd = smem + KV_OFF + (c & 1) * KV_BUF + KC * D * 2;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (16 * u < KW) {
            uint32_t ph[4], pl[4];
            ptx::split_bf16(sacc[2 * u][0], sacc[2 * u][1], ph[0], pl[0]);
            ptx::split_bf16(sacc[2 * u][2], sacc[2 * u][3], ph[1], pl[1]);
            ptx::split_bf16(sacc[2 * u + 1][0], sacc[2 * u + 1][1], ph[2], pl[2]);
            ptx::split_bf16(sacc[2 * u + 1][2], sacc[2 * u + 1][3], ph[3], pl[3]);
            const int vrow = sp * KW + 16 * u + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
            for (int dp = 0; dp < 8; ++dp) {
              uint32_t vb[4];
              ptx::ldmatrix_x4_trans(vb, vd + swz(vrow, 2 * dp + (lane >> 4)));
              ptx::mma_bf16_16816(oacc[2 * dp], ph, vb);
              ptx::mma_bf16_16816(oacc[2 * dp + 1], ph, vb + 2);
              ptx::mma_bf16_16816(oacc[2 * dp], pl, vb);
              ptx::mma_bf16_16816(oacc[2 * dp + 1], pl, vb + 2);
            }
          }
        }
      }
      __syncthreads();
      // attention mass of this chunk's keys, summed over m-tiles in order
      if (part && tid < KC) {
        const int j = c * KC + tid;
        if (j < nk) {
          float s = 0.f;
          for (int m2 = 0; m2 < n_mt; ++m2) s += massb[m2 * KC + tid];
          const int slot = (j < L) ? j : ctrl->row_slot[xrow[j - L]];
          part[slot] = s;
        }
      }
    }
    // -------------------------------------------- combine O over key splits
    float* obuf = reinterpret_cast<float*>(smem + OBUF_OFF);
    if (active) {
      float* ow = obuf + warp * 16 * OBUF_LD;
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        *reinterpret_cast<float2*>(ow + gq * OBUF_LD + 8 * t + 2 * qd) =
            make_float2(oacc[t][0], oacc[t][1]);
        *reinterpret_cast<float2*>(ow + (gq + 8) * OBUF_LD + 8 * t + 2 * qd) =
            make_float2(oacc[t][2], oacc[t][3]);
      }
    }
    __syncthreads();
    for (int idx = tid; idx < n * (D / 4); idx += NTHREADS) {
      const int r = idx / (D / 4);
      const int d4 = (idx % (D / 4)) * 4;
      const int mt2 = r >> 4, rr = r & 15;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s2 = 0; s2 < n_split; ++s2) {
        const float4 v =
            *reinterpret_cast<const float4*>(obuf + (s2 * n_mt + mt2) * 16 * OBUF_LD + rr * OBUF_LD + d4);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      *reinterpret_cast<float4*>(a.out + (size_t)(row0 + ra + r) * H + h * D + d4) = acc;
    }
    __syncthreads();
  }
}

}  // namespace

size_t step_bf16_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_step_bf16(const StepPlan& plan, const StepArgs& a, const void* tmap_x,
                             const void* tmap_w, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(step_bf16_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int grid = plan.n_groups * a.n_heads;
  if (grid == 0) return cudaSuccess;
  step_bf16_kernel<<<grid, NTHREADS, SMEM_BYTES, stream>>>(
      plan, a, *reinterpret_cast<const CUtensorMap*>(tmap_x),
      *reinterpret_cast<const CUtensorMap*>(tmap_w));
  return cudaGetLastError();
}

}  // namespace fdllm
