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
// Phase 1 (projection): [128 rows x H] x [H x 384], the 384 columns being
//   this head's q | k | v blocks of Wqkv. TMA streams x and Wqkv tiles
//   (128-byte swizzle) through a 3-stage mbarrier pipeline; one thread
//   issues tcgen05.mma (M=128, N=128, K=16, bf16 -> fp32) into TMEM.
// Phase 2 (epilogue): all 8 warps read the accumulator from TMEM, apply
//   rotate-half RoPE to q and k, round to bf16, keep q in shared memory in
//   the UMMA operand layout, and copy k/v rows to their cache slots with
//   coalesced 16-byte stores.
// Phase 3 (attention), per sequence of the group, on the tensor cores in
//   transposed form so that a sequence of only 16..128 rows wastes no MMA
//   rows: S^T = K Q^T (keys on TMEM lanes, the sequence's rows on columns)
//   and O^T += V^T P^T. K and V pages are gathered by TMA through the block
//   table, two 64-slot pages per 128-key chunk, into a 3-slot ring.
//   Pass 1 finds every row's log-sum-exp (column max/sum across the 128
//   key lanes by a shuffle reduce-scatter); pass 2 forms the exact
//   probabilities, whose per-key sums over the rows are the attention mass
//   (one thread per key, no cross-thread reduction), and feeds P^T to the
//   P.V product as bf16 hi + lo parts. The Flash-Verify two-view rule
//   (paragraph 3 of the same page) decides visibility of fresh view keys.
#include <cuda.h>
#include <cuda_bf16.h>

#include "fdllm_internal.h"
#include "ptx.cuh"

namespace fdllm {
namespace {

constexpr int D = 128;            // head_dim served by this kernel
constexpr int BM = 128;           // rows per group (UMMA M of the projection)
constexpr int BK = 64;            // K per pipeline stage (one 128-byte swizzle span)
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;           // 16 KB
constexpr int BOX_BYTES = BK * 64 * 2;         // 8 KB: 64 K-rows x 64 columns
constexpr int B_BYTES = 6 * BOX_BYTES;         // q, k, v blocks, two boxes each
constexpr int STAGE_BYTES = A_BYTES + B_BYTES; // 64 KB
constexpr int PIPE_BYTES = STAGES * STAGE_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int NTHREADS = 256;
constexpr int PS = 64;                          // cache page size served
constexpr int MAX_PAGES = 512;                  // logical pages per sequence
constexpr uint64_t WAIT_NS = 1000000000ull;     // bounded waits: 1 s

// Reuse of the pipeline area after the projection.
constexpr int Q_OFF = 0;              // q: [2 d-halves][128 rows][128 B], K-major SW128
constexpr int HALF_BYTES = 16384;     // one d-half of a 128-row (or 128-key) operand
constexpr int KST_OFF = 32768;        // fresh k rows staged for the cache copy
constexpr int VST_OFF = 65536;        // fresh v rows staged for the cache copy
constexpr int SLOT_OFF = 32768;       // attention ring: 3 slots of a 128-key K or V chunk
constexpr int SLOT_BYTES = 32768;     //   [2 d-halves][128 keys][128 B], SW128 (TMA layout)
constexpr int NSLOT = 3;
constexpr int PT_OFF = SLOT_OFF + NSLOT * SLOT_BYTES;   // P^T hi, then lo
constexpr int PT_BYTES = 32768;       //   core matrices: [rows/8][128 keys][16 B]
static_assert(PT_OFF + 2 * PT_BYTES <= PIPE_BYTES, "attention buffers overflow");

// TMEM columns during attention.
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256;

struct Ctrl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t mma_done;
  uint64_t afull[NSLOT];
  uint64_t aempty[NSLOT];
  uint64_t s_full[2];
  uint64_t s_empty[2];
  uint64_t p_full;
  uint64_t pv_done;
  uint64_t o_done;
  uint32_t tmem_base;
  int abort;
  // per-row metadata of the group
  int row_pos[BM];
  int row_slot[BM];
  int row_page[BM];       // -1: row has bad metadata
  int row_view[BM];
  int row_q[BM];          // row of q in shared memory (sequences padded to 16 rows)
  // current sequence
  int nx, npages;
  int xs_slot[BM];        // slots written by view rows, ascending
  int xs_row[BM];         // their group rows
  int pg_log[MAX_PAGES];  // logical pages attended, in order
  int pg_phys[MAX_PAGES]; // physical page, -1 when the table entry is bad
  float m_run[BM], l_run[BM], mnew[BM], lse2[BM];
  float red[4][BM];
};
constexpr int CTRL_OFF = PIPE_BYTES;
constexpr int SMEM_BYTES = PIPE_BYTES + (int)sizeof(Ctrl) + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

__device__ __forceinline__ void set_err(int* err, int code, int detail) {
  if (atomicCAS(err, 0, code) == 0) err[1] = detail;
}

// Bounded wait that records a timeout once and then stops waiting (sticky),
// so every role still walks through its remaining synchronisation points.
__device__ __forceinline__ bool wait_bar(Ctrl* c, uint64_t* bar, uint32_t parity, int* err,
                                         int site) {
  if (*reinterpret_cast<volatile int*>(&c->abort)) return false;
  if (ptx::mbar_wait(bar, parity, WAIT_NS)) return true;
  set_err(err, kDevTimeout, site);
  atomicExch(&c->abort, 1);
  return false;
}

// 128-byte swizzled K-major operand: byte offset of the 16-byte chunk `ch`
// (0..7) of row `r` inside one d-half.
__device__ __forceinline__ uint32_t sw128(int r, int ch) {
  return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
}

// Fresh k/v staging rows (256 bytes each, 16-byte chunks XOR-swizzled).
__device__ __forceinline__ uint32_t swz256(int row, int chunk) {
  return (uint32_t)(row * 256 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Reduce-scatter of 32 columns over the 32 lanes: afterwards v[0] of lane l
// holds the max (or sum) over all lanes of column l.
template <bool kMax>
__device__ __forceinline__ float reduce_scatter32(float* v, int lane) {
#pragma unroll
  for (int k = 16; k >= 1; k >>= 1) {
    const bool upper = (lane & k) != 0;
#pragma unroll
    for (int i = 0; i < k; ++i) {
      const float send = upper ? v[i] : v[i + k];
      const float keep = upper ? v[i + k] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, k);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  return v[0];
}

__device__ __forceinline__ void rope32(float* lo, float* hi, int pos, int c, const float* cos_t,
                                       const float* sin_t) {
  const float4* cp = reinterpret_cast<const float4*>(cos_t + (size_t)pos * (D / 2) + 32 * c);
  const float4* sp = reinterpret_cast<const float4*>(sin_t + (size_t)pos * (D / 2) + 32 * c);
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const float4 cs = __ldg(cp + u), sn = __ldg(sp + u);
    const float cv[4] = {cs.x, cs.y, cs.z, cs.w}, sv[4] = {sn.x, sn.y, sn.z, sn.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int t = 4 * u + e;
      const float a = lo[t], b = hi[t];
      lo[t] = a * cv[e] - b * sv[e];
      hi[t] = b * cv[e] + a * sv[e];
    }
  }
}

__device__ __forceinline__ uint4 pack8(const float* v) {
  uint4 w;
  w.x = ptx::pack_bf16(v[0], v[1]);
  w.y = ptx::pack_bf16(v[2], v[3]);
  w.z = ptx::pack_bf16(v[4], v[5]);
  w.w = ptx::pack_bf16(v[6], v[7]);
  return w;
}

// TMEM -> registers -> RoPE -> bf16 -> q operand rows. Every lane of the
// warp executes the TMEM loads; only valid rows are rotated and written.
__device__ __forceinline__ void epi_q(uint32_t taddr, int qrow, bool valid, int pos,
                                      const float* cos_t, const float* sin_t, uint8_t* q) {
#pragma unroll 1
  for (int c = 0; c < 2; ++c) {
    float lo[32], hi[32];
    ptx::tmem_ld32(taddr + 32 * c, lo);
    ptx::tmem_ld32(taddr + 64 + 32 * c, hi);
    ptx::tmem_ld_wait();
    if (!valid) continue;
    rope32(lo, hi, pos, c, cos_t, sin_t);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      *reinterpret_cast<uint4*>(q + sw128(qrow, 4 * c + u)) = pack8(lo + 8 * u);
      *reinterpret_cast<uint4*>(q + HALF_BYTES + sw128(qrow, 4 * c + u)) = pack8(hi + 8 * u);
    }
  }
}

// k (rotated) or v (plain) rows -> bf16 staging rows for the cache copy.
__device__ __forceinline__ void epi_kv(uint32_t taddr, int row, bool valid, bool rotate, int pos,
                                       const float* cos_t, const float* sin_t, uint8_t* dst) {
#pragma unroll 1
  for (int c = 0; c < 2; ++c) {
    float lo[32], hi[32];
    ptx::tmem_ld32(taddr + 32 * c, lo);
    ptx::tmem_ld32(taddr + 64 + 32 * c, hi);
    ptx::tmem_ld_wait();
    if (!valid) continue;
    if (rotate) rope32(lo, hi, pos, c, cos_t, sin_t);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      *reinterpret_cast<uint4*>(dst + swz256(row, 4 * c + u)) = pack8(lo + 8 * u);
      *reinterpret_cast<uint4*>(dst + swz256(row, 8 + 4 * c + u)) = pack8(hi + 8 * u);
    }
  }
}

__global__ void __launch_bounds__(NTHREADS, 1)
    step_bf16_kernel(const __grid_constant__ StepPlan plan, const __grid_constant__ StepArgs a,
                     const __grid_constant__ CUtensorMap tmap_x,
                     const __grid_constant__ CUtensorMap tmap_w,
                     const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v) {
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
  const int layer = plan.layer;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&ctrl->full[s], 1);
      ptx::mbar_init(&ctrl->empty[s], 1);
    }
    for (int s = 0; s < NSLOT; ++s) {
      ptx::mbar_init(&ctrl->afull[s], 1);
      ptx::mbar_init(&ctrl->aempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&ctrl->s_full[s], 1);
      ptx::mbar_init(&ctrl->s_empty[s], 4);
    }
    ptx::mbar_init(&ctrl->mma_done, 1);
    ptx::mbar_init(&ctrl->p_full, 4);
    ptx::mbar_init(&ctrl->pv_done, 1);
    ptx::mbar_init(&ctrl->o_done, 1);
    ctrl->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&ctrl->tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (tid == 64) {
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_k);
    ptx::prefetch_tmap(&tmap_v);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;

  // ================================================================ projection
  if (warp == 0) {
    if (lane == 0) {   // TMA producer
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES;
        const int u = kb / STAGES;
        if (u > 0 && !wait_bar(ctrl, &ctrl->empty[s], (u - 1) & 1, a.err, 1)) break;
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
    if (lane == 0) {   // MMA issuer
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(BM, 128, false, true);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES;
        const int u = kb / STAGES;
        if (!wait_bar(ctrl, &ctrl->full[s], u & 1, a.err, 2)) break;
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
    // row metadata (warps 2..7)
    for (int i = tid - 64; i < BM; i += NTHREADS - 64) {
      int pos = 0, slot = 0, page = -1, view = 0, qr = 0;
      if (i < nrows) {
        const int gr = row0 + i;
        pos = a.positions[gr];
        slot = a.slots ? a.slots[gr] : pos;
        view = a.view ? (int)a.view[gr] : 0;
        int b = seq_a;
        while (b + 1 < seq_b && plan.cu_rows[b + 1] <= gr) ++b;
        qr = plan.seq_qoff[b] + (gr - plan.cu_rows[b]);
        if (pos < 0 || pos >= a.max_position) {
          set_err(a.err, kDevBadPosition, gr);
        } else if (slot < 0 || slot >= plan.row_stride) {
          set_err(a.err, kDevBadSlot, gr);
        } else {
          const int pg = a.block_table[(size_t)b * plan.max_blocks + slot / PS];
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
      ctrl->row_q[i] = qr;
    }
  }
  __syncwarp();
  __syncthreads();   // row metadata visible; producer and MMA loops issued

  // ================================================================ epilogue
  const bool acc_ok = wait_bar(ctrl, &ctrl->mma_done, 0, a.err, 3);
  __syncwarp();
  ptx::tc_fence_after();
  {
    const int quad = warp & 3;
    const int i = quad * 32 + lane;
    const bool valid = acc_ok && i < nrows && ctrl->row_page[i] >= 0;
    const int pos = ctrl->row_pos[i];
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    if (warp < 4) {
      epi_q(trow + 0, ctrl->row_q[i], valid, pos, a.rope_cos, a.rope_sin, smem + Q_OFF);
    } else {
      epi_kv(trow + 128, i, valid, true, pos, a.rope_cos, a.rope_sin, smem + KST_OFF);
      epi_kv(trow + 256, i, valid, false, pos, a.rope_cos, a.rope_sin, smem + VST_OFF);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();

  // Fresh k/v rows -> cache slots (16 consecutive threads per 256-byte row).
  {
    const size_t head_stride = (size_t)PS * D;
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
                         (size_t)(slot % PS) * D + ch * 8;
      const uint8_t* src = smem + (part < 16 ? KST_OFF : VST_OFF) + swz256(r, ch);
      __nv_bfloat16* dst = (part < 16 ? kp : vp) + off;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    }
  }
  // The cache writes must be visible to this CTA's TMA reads, and the q
  // operand written by st.shared to the tensor cores.
  asm volatile("fence.proxy.async.global;" ::: "memory");
  fence_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();

  // ================================================================ attention
  const float sl2 = 1.4426950408889634f * rsqrtf((float)D);   // log2(e) / sqrt(D)
  const uint32_t q_base = ptx::smem_u32(smem + Q_OFF);
  const uint32_t slot_base = ptx::smem_u32(smem + SLOT_OFF);
  const uint32_t pt_base = ptx::smem_u32(smem + PT_OFF);
  // Schedule counters, identical in every thread: chunk loads (K or V)
  // issued so far, S^T products, P.V products, finished sequences.
  uint32_t ring = 0, scount = 0, pcount = 0, ocount = 0;

  for (int b = seq_a; b < seq_b; ++b) {
    const int n = plan.cu_rows[b + 1] - plan.cu_rows[b];
    if (n == 0) continue;
    const int ra = plan.cu_rows[b] - row0;
    const int L = plan.seq_lens[b];
    const int N16 = (n + 15) & ~15;
    const int qoff = plan.seq_qoff[b];
    const int nblk = (N16 + 31) >> 5;

    // ---------------------------------------- sequence setup (all threads)
    // view rows with good metadata, sorted by slot
    if (tid < n) {
      const int i = ra + tid;
      if (ctrl->row_view[i] != 0 && ctrl->row_page[i] >= 0) {
        const int si = ctrl->row_slot[i];
        int rank = 0;
        for (int j = 0; j < n; ++j) {
          const int jj = ra + j;
          if (ctrl->row_view[jj] == 0 || ctrl->row_page[jj] < 0) continue;
          const int sj = ctrl->row_slot[jj];
          rank += (sj < si || (sj == si && j < tid)) ? 1 : 0;
        }
        ctrl->xs_slot[rank] = si;
        ctrl->xs_row[rank] = i;
      }
    }
    const int nx = __syncthreads_count(tid < n && ctrl->row_view[ra + tid] != 0 &&
                                       ctrl->row_page[ra + tid] >= 0);
    const int npr = min((L + PS - 1) / PS, MAX_PAGES);
    for (int i = tid; i < npr; i += NTHREADS) ctrl->pg_log[i] = i;
    if (tid == 0) {
      int np = npr;
      int last = -1;
      for (int t = 0; t < nx; ++t) {
        const int p = ctrl->xs_slot[t] / PS;
        if (p >= npr && p != last && np < MAX_PAGES) {
          ctrl->pg_log[np++] = p;
          last = p;
        }
      }
      ctrl->npages = np;
    }
    __syncthreads();
    const int npages = ctrl->npages;
    const int* bt = a.block_table + (size_t)b * plan.max_blocks;
    for (int i = tid; i < npages; i += NTHREADS) {
      const int pg = bt[ctrl->pg_log[i]];
      if (pg < 0 || pg >= a.num_pages) {
        set_err(a.err, kDevBadPage, -1 - ctrl->pg_log[i]);
        ctrl->pg_phys[i] = -1;
      } else {
        ctrl->pg_phys[i] = pg;
      }
    }
    if (tid < BM) {
      ctrl->m_run[tid] = -INFINITY;
      ctrl->l_run[tid] = 0.f;
    }
    __syncthreads();
    const int nch = (npages + 1) >> 1;
    bool any_page = false;
    for (int i = 0; i < npages; ++i) any_page |= ctrl->pg_phys[i] >= 0;
    float* part = a.mass_part ? a.mass_part + ((size_t)h * plan.batch + b) * plan.row_stride
                              : nullptr;
    // Chunk loads of this sequence: pass 1 K_0..K_{nch-1} (items r0 + c),
    // pass 2 K_c, V_c (items r0 + nch + 2c, r0 + nch + 2c + 1).
    const uint32_t r0 = ring, s0 = scount, p0 = pcount;

    if (warp == 0) {
      // ---------------------------------------- TMA producer
      if (lane == 0) {
        uint32_t item = r0;
        for (int pass = 0; pass < 2; ++pass) {
          for (int c = 0; c < nch; ++c) {
            for (int which = 0; which <= pass; ++which, ++item) {
              const int s = item % NSLOT;
              const uint32_t u = item / NSLOT;
              if (u > 0) wait_bar(ctrl, &ctrl->aempty[s], (u - 1) & 1, a.err, 10);
              uint32_t bytes = 0;
              int phys[2] = {-1, -1};
              for (int pi = 0; pi < 2; ++pi) {
                const int pidx = 2 * c + pi;
                if (pidx < npages && ctrl->pg_phys[pidx] >= 0) {
                  phys[pi] = ctrl->pg_phys[pidx];
                  bytes += 2 * BOX_BYTES;
                }
              }
              ptx::mbar_arrive_expect_tx(&ctrl->afull[s], bytes);
              uint8_t* dst = smem + SLOT_OFF + s * SLOT_BYTES;
              const CUtensorMap* map = which == 0 ? &tmap_k : &tmap_v;
              for (int pi = 0; pi < 2; ++pi) {
                if (phys[pi] < 0) continue;
                const int row = ((layer * a.num_pages + phys[pi]) * a.n_heads + h) * PS;
                ptx::tma_load_2d(dst + pi * BOX_BYTES, map, 0, row, &ctrl->afull[s]);
                ptx::tma_load_2d(dst + HALF_BYTES + pi * BOX_BYTES, map, 64, row, &ctrl->afull[s]);
              }
            }
          }
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------- MMA issuer
      if (lane == 0) {
        const uint32_t idesc_s = ptx::idesc_bf16_f32(128, N16, false, false);
        const uint32_t idesc_pv = ptx::idesc_bf16_f32(128, N16, true, true);
        // S^T number j of this sequence from chunk-load item `item`.
        auto issue_s = [&](uint32_t j, uint32_t item) {
          const int s = item % NSLOT;
          wait_bar(ctrl, &ctrl->afull[s], (item / NSLOT) & 1, a.err, 11);
          const uint32_t idx = s0 + j;
          const uint32_t sb = idx & 1, su = idx >> 1;
          if (su > 0) wait_bar(ctrl, &ctrl->s_empty[sb], (su - 1) & 1, a.err, 12);
          ptx::tc_fence_after();
          const uint32_t kbase = slot_base + s * SLOT_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
            // A: K chunk, K-major, M = 128 keys; B: q rows, K-major, N = N16.
            const uint64_t ad = ptx::smem_desc_sw128(kbase + off, 16, 1024);
            const uint64_t bd = ptx::smem_desc_sw128(q_base + off + qoff * 128, 16, 1024);
            ptx::umma_f16_ss(tmem + (sb ? TM_S1 : TM_S0), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          ptx::umma_commit(&ctrl->s_full[sb]);
          ptx::umma_commit(&ctrl->aempty[s]);
        };
        for (int c = 0; c < nch; ++c) issue_s(c, r0 + c);
        bool any = false;
        if (nch > 0) issue_s(nch, r0 + nch);
        for (int c = 0; c < nch; ++c) {
          if (c + 1 < nch) issue_s(nch + c + 1, r0 + nch + 2 * (c + 1));
          const uint32_t vitem = r0 + nch + 2 * c + 1;
          const int vs = vitem % NSLOT;
          wait_bar(ctrl, &ctrl->afull[vs], (vitem / NSLOT) & 1, a.err, 13);
          wait_bar(ctrl, &ctrl->p_full, (p0 + c) & 1, a.err, 14);
          ptx::tc_fence_after();
          const uint32_t vbase = slot_base + vs * SLOT_BYTES;
          for (int pi = 0; pi < 2; ++pi) {
            const int pidx = 2 * c + pi;
            if (pidx >= npages || ctrl->pg_phys[pidx] < 0) continue;
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const int ks = pi * 4 + k4;   // 16 keys per step
              // A = V^T: M = d, N-major in shared memory (64 d per 128-byte
              // row), two 64-d blocks 16 KB apart (LBO), 8-key groups 1 KB
              // apart (SBO).
              const uint64_t ad = ptx::smem_desc_sw128(vbase + ks * 2048, HALF_BYTES, 1024);
              // B = P^T: N-major core matrices without swizzle: 8-key
              // groups 128 B apart (LBO), 8-row blocks 2048 B apart (SBO).
              const uint64_t bh = ptx::smem_desc_noswz(pt_base + ks * 256, 128, 2048);
              const uint64_t bl = ptx::smem_desc_noswz(pt_base + PT_BYTES + ks * 256, 128, 2048);
              ptx::umma_f16_ss(tmem + TM_O, ad, bh, idesc_pv, any ? 1u : 0u);
              ptx::umma_f16_ss(tmem + TM_O, ad, bl, idesc_pv, 1u);
              any = true;
            }
          }
          ptx::umma_commit(&ctrl->aempty[vs]);
          ptx::umma_commit(&ctrl->pv_done);
        }
        ptx::umma_commit(&ctrl->o_done);
      }
    } else if (warp >= 4) {
      // ---------------------------------------- softmax warps: one key per thread
      const int t = tid - 128;                 // key lane in a 128-key chunk, d lane for O^T
      const int quad = warp - 4;
      const uint32_t tl = (uint32_t)(quad * 32) << 16;
      // cat: 0 nobody attends the key, 1 every row does, 2 a view row's slot
      auto key_info = [&](int c, int& slot, int& cat, int& xr) {
        const int pidx = 2 * c + (t >> 6);
        cat = 0;
        xr = -1;
        slot = -1;
        if (pidx >= npages || ctrl->pg_phys[pidx] < 0) return;
        slot = ctrl->pg_log[pidx] * PS + (t & 63);
        if (slot < L) {
          cat = 1;
          return;
        }
        int lo = 0, hi = nx - 1;
        while (lo <= hi) {
          const int mid = (lo + hi) >> 1;
          const int v = ctrl->xs_slot[mid];
          if (v == slot) {
            cat = 2;
            xr = ctrl->xs_row[mid];
            return;
          }
          if (v < slot) lo = mid + 1; else hi = mid - 1;
        }
      };
      auto visible = [&](int cat, int xr, int col) -> bool {
        if (col >= n) return false;
        if (cat == 1) return true;
        if (cat == 0) return false;
        const int rr = ra + col;
        const int vr = ctrl->row_view[rr];
        return vr != 0 && vr == ctrl->row_view[xr] && ctrl->row_pos[xr] <= ctrl->row_pos[rr];
      };

      // ----- pass 1: log-sum-exp of every row
      for (int c = 0; c < nch; ++c) {
        int slot, cat, xr;
        key_info(c, slot, cat, xr);
        const uint32_t idx = s0 + c;
        const uint32_t sb = idx & 1;
        wait_bar(ctrl, &ctrl->s_full[sb], (idx >> 1) & 1, a.err, 20);
        ptx::tc_fence_after();
        const uint32_t sbase = tmem + tl + (sb ? TM_S1 : TM_S0);
        for (int blk = 0; blk < nblk; ++blk) {
          float v[32];
          ptx::tmem_ld32(sbase + 32 * blk, v);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            v[j] = visible(cat, xr, 32 * blk + j) ? v[j] * sl2 : -INFINITY;
          ctrl->red[quad][32 * blk + lane] = reduce_scatter32<true>(v, lane);
        }
        named_bar(1, 128);
        if (t < N16) {
          const float cm = fmaxf(fmaxf(ctrl->red[0][t], ctrl->red[1][t]),
                                 fmaxf(ctrl->red[2][t], ctrl->red[3][t]));
          ctrl->mnew[t] = fmaxf(ctrl->m_run[t], cm);
        }
        named_bar(1, 128);
        for (int blk = 0; blk < nblk; ++blk) {
          float v[32];
          ptx::tmem_ld32(sbase + 32 * blk, v);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int col = 32 * blk + j;
            v[j] = visible(cat, xr, col) ? exp2f(v[j] * sl2 - ctrl->mnew[col]) : 0.f;
          }
          ctrl->red[quad][32 * blk + lane] = reduce_scatter32<false>(v, lane);
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&ctrl->s_empty[sb]);
        named_bar(1, 128);
        if (t < N16) {
          const float mn = ctrl->mnew[t];
          const float sm = ctrl->red[0][t] + ctrl->red[1][t] + ctrl->red[2][t] + ctrl->red[3][t];
          if (mn != -INFINITY) ctrl->l_run[t] = ctrl->l_run[t] * exp2f(ctrl->m_run[t] - mn) + sm;
          ctrl->m_run[t] = mn;
        }
        named_bar(1, 128);
      }
      if (t < N16)
        ctrl->lse2[t] = ctrl->l_run[t] > 0.f ? ctrl->m_run[t] + log2f(ctrl->l_run[t]) : INFINITY;
      // mass row past the context: zero (view slots are written below)
      if (part)
        for (int j = L + t; j < plan.row_stride; j += 128) part[j] = 0.f;
      named_bar(1, 128);

      // ----- pass 2: probabilities, mass, P^T for the P.V product
      for (int c = 0; c < nch; ++c) {
        int slot, cat, xr;
        key_info(c, slot, cat, xr);
        const int pidx = 2 * c + (t >> 6);
        const bool loaded = pidx < npages && ctrl->pg_phys[pidx] >= 0;
        const uint32_t idx = s0 + nch + c;
        const uint32_t sb = idx & 1;
        wait_bar(ctrl, &ctrl->s_full[sb], (idx >> 1) & 1, a.err, 21);
        ptx::tc_fence_after();
        const uint32_t sbase = tmem + tl + (sb ? TM_S1 : TM_S0);
        uint32_t ph[4][16], pl[4][16];
        float mass = 0.f;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          if (blk < nblk) {
            float v[32];
            ptx::tmem_ld32(sbase + 32 * blk, v);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const int col = 32 * blk + j;
              const float q0 = visible(cat, xr, col) ? exp2f(v[j] * sl2 - ctrl->lse2[col]) : 0.f;
              const float q1 =
                  visible(cat, xr, col + 1) ? exp2f(v[j + 1] * sl2 - ctrl->lse2[col + 1]) : 0.f;
              mass += q0 + q1;
              ptx::split_bf16(q0, q1, ph[blk][j >> 1], pl[blk][j >> 1]);
            }
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&ctrl->s_empty[sb]);
        if (part && cat != 0) part[slot] = mass;
        // V rows of keys nobody attends may hold anything (page tails):
        // zero them so that 0 * V stays 0 in the P.V product.
        const uint32_t vitem = r0 + nch + 2 * c + 1;
        const int vs = vitem % NSLOT;
        if (loaded && cat == 0) {
          wait_bar(ctrl, &ctrl->afull[vs], (vitem / NSLOT) & 1, a.err, 22);
          uint8_t* vrow = smem + SLOT_OFF + vs * SLOT_BYTES + (t >> 6) * BOX_BYTES + (t & 63) * 128;
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            *reinterpret_cast<uint4*>(vrow + ch * 16) = z;
            *reinterpret_cast<uint4*>(vrow + HALF_BYTES + ch * 16) = z;
          }
        }
        // The P^T buffers are free once the previous P.V product completed.
        const uint32_t pidx_g = p0 + c;
        if (pidx_g > 0) wait_bar(ctrl, &ctrl->pv_done, (pidx_g - 1) & 1, a.err, 23);
        uint8_t* pth = smem + PT_OFF;
        uint8_t* ptl = pth + PT_BYTES;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          if (blk < nblk) {
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
              const int nb = 4 * blk + g8;     // 8-row block of the sequence
              if (8 * nb < N16) {
                *reinterpret_cast<uint4*>(pth + nb * 2048 + t * 16) =
                    make_uint4(ph[blk][4 * g8], ph[blk][4 * g8 + 1], ph[blk][4 * g8 + 2],
                               ph[blk][4 * g8 + 3]);
                *reinterpret_cast<uint4*>(ptl + nb * 2048 + t * 16) =
                    make_uint4(pl[blk][4 * g8], pl[blk][4 * g8 + 1], pl[blk][4 * g8 + 2],
                               pl[blk][4 * g8 + 3]);
              }
            }
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&ctrl->p_full);
      }
      // ----- O^T -> out (thread t = head dimension t)
      wait_bar(ctrl, &ctrl->o_done, ocount & 1, a.err, 24);
      ptx::tc_fence_after();
      for (int blk = 0; blk < nblk; ++blk) {
        float v[32];
        ptx::tmem_ld32(tmem + tl + TM_O + 32 * blk, v);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int r = 32 * blk + j;
          if (r < n) a.out[(size_t)(row0 + ra + r) * H + h * D + t] = any_page ? v[j] : 0.f;
        }
      }
      ptx::tc_fence_before();
    }
    ring = r0 + 3 * nch;
    scount = s0 + 2 * nch;
    pcount = p0 + nch;
    ++ocount;
    __syncwarp();
    __syncthreads();
  }

  // ================================================================ teardown
  if (warp == 1 && lane == 0) {
    // every tcgen05 operation issued by this thread has completed
    ptx::umma_commit(&ctrl->mma_done);
    ptx::mbar_wait(&ctrl->mma_done, 1, WAIT_NS);
  }
  if (warp == 0 && lane == 0 && ring > 0) {
    // the last chunk loads have landed (they have, unless a wait timed out)
    for (uint32_t it = ring > NSLOT ? ring - NSLOT : 0; it < ring; ++it)
      ptx::mbar_wait(&ctrl->afull[it % NSLOT], (it / NSLOT) & 1, WAIT_NS);
  }
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) ptx::tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace

size_t step_bf16_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_step_bf16(const StepPlan& plan, const StepArgs& a, const void* tmap_x,
                             const void* tmap_w, const void* tmap_k, const void* tmap_v,
                             cudaStream_t stream) {
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
      *reinterpret_cast<const CUtensorMap*>(tmap_w), *reinterpret_cast<const CUtensorMap*>(tmap_k),
      *reinterpret_cast<const CUtensorMap*>(tmap_v));
  return cudaGetLastError();
}

}  // namespace fdllm
