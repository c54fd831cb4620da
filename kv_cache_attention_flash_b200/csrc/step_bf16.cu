// Flash-Cache fused layer step for bf16 on sm_100a.
//
// The unit of work is a tile: one (row group g, head h). A row group packs
// whole sequences into at most 128 query rows, so every fresh key/value a
// sequence attends to is produced by the CTA that attends to it, and no
// grid-wide ordering is needed ("Flash-dLLM: I/O-Aware KV Caching and
// Parallel Decoding for Fast, Memory-Efficient Diffusion LLMs", ai4snews
// summary, paragraph 1: QKV projection, RoPE and the cache write fused, K/V
// written to the cache from on-chip memory; scheduled attention aligns each
// query block with its own KV blocks through a block table). The kernel
// runs one CTA per tile, or, when the tiles outnumber the SMs, one
// persistent CTA per SM over a host-built list of tiles (kPersist); then
// barrier phases, schedule counters and the TMEM allocation carry over from
// tile to tile. TMA loads carry L2 eviction hints: x rows, Wqkv slices and
// pass-1 K chunks are read again and stay; pass-2 K and V go first.
//
// Phase 1 (projection): [128 rows x H] x [H x 384], the 384 columns being
//   this head's q | k | v blocks of Wqkv. TMA streams x and Wqkv tiles
//   (128-byte swizzle) through a 3-stage mbarrier pipeline; one thread
//   issues tcgen05.mma (M=128, N=256 for q|k and N=128 for v, K=16,
//   bf16 -> fp32) into TMEM.
// Phase 2 (epilogue): all 8 warps read the accumulator from TMEM, apply
//   rotate-half RoPE to q and k, round to bf16, keep q in shared memory in
//   the UMMA operand layout, and copy k/v rows to their cache slots with
//   coalesced 16-byte stores.
// Phase 3 (attention), per sequence of the group, on the tensor cores. K
//   and V pages are gathered by TMA through the block table, two 64-slot
//   pages per 128-key chunk, into a 3-slot ring. A sequence of 16, 32 or 64
//   padded rows whose chunks' scores fit the 512 TMEM columns keeps them
//   resident: one S^T = K Q^T product per chunk, K read once, row maxima and
//   sums reduced across lanes and lane quadrants, P formed from the same
//   scores. Any other sequence takes two passes:
//   Pass 1 finds every row's log-sum-exp from S = Q K^T with the rows on
//   TMEM lanes, so each thread keeps its own row's running max and sum. A
//   sequence of at most 64 rows is first repeated across the four lane
//   quadrants, each copy taking a share of every chunk's keys, so that all
//   four SM sub-partitions share its exponentials; the two warps of a
//   quadrant split the copy's keys, and the partial pairs merge at the end.
//   Pass 2 runs in transposed form so that a sequence of only 16..128 rows
//   wastes no MMA rows: S^T = K Q^T (keys on lanes, the sequence's rows on
//   columns) gives the exact probabilities, whose per-key sums over the
//   rows are the attention mass (one thread per key, no cross-thread
//   reduction), and O^T += V^T P^T takes P^T as bf16 hi + lo parts, the lo
//   rows stacked after the hi rows so that one product of twice the width
//   accumulates both (O^T hi and lo in adjacent column ranges, summed when
//   out is stored). The
//   Flash-Verify two-view rule (paragraph 3 of the same page) decides
//   visibility of fresh view keys, read from a table the tile builds once
//   (one 32-bit word per view slot and 32 rows).
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstddef>
#include <type_traits>

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
// A split tile's CTA loads one of the q, k, v blocks (a third of B): its
// 32 KB stages make a ring twice as deep in the same bytes.
// Cluster split-K (few tiles): each of the 4 CTAs of a tile's cluster
// accumulates q | k | v over a quarter of the K range; the partials meet in
// the owners' shared memory (q: rank 0, k: rank 1, v: rank 2), one fp32
// [32 column quads][128 rows][4] slot of 64 KB per sending rank.
constexpr int CL_RANKS = 4;
constexpr int CL_SLOT_BYTES = 65536;
static_assert(3 * CL_SLOT_BYTES <= PIPE_BYTES, "cluster partial slots");
constexpr int TMEM_COLS = 512;
constexpr int NTHREADS = 320;        // warps 0-7: epilogue / softmax (two per TMEM quadrant),
                                      // warp 8: TMA producer, warp 9: MMA issuer and TMEM owner
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int NSMX = 256;             // threads of warps 0-7
constexpr int PS = 64;                          // cache page size served
constexpr int MAX_PAGES = 1024;                 // logical pages attended per row group
constexpr int MAX_SEQ = 8;                      // sequences per row group (16 padded rows each)
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
// A sequence of at most 64 rows keeps P^T lo at PT_OFF + 16 KB; the last
// 32 KB then hold its q rows repeated across the four TMEM lane quadrants
// for pass 1.
constexpr int QREP_OFF = PT_OFF + 32768;

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
  uint64_t q_ready;       // repeated q rows written (sequences of at most 64 rows)
  uint64_t o_done;
  uint64_t s_half;        // resident scores: the first half of the chunks' S^T is in TMEM
  uint64_t s_all;         //   and all of them (each completes once per sequence)
  uint64_t t_free;        // the softmax warps are done with this sequence's TMEM
  uint64_t pv_buf[2];     // resident scores: P.V product done with P^T buffer 0 / 1
  uint64_t p_buf[2];      //   and P^T buffer 0 / 1 written (8 softmax warps)
  uint64_t kv_ready;      // cluster split-K, rank 0: the k and v owners' rows are in the cache
  uint32_t tmem_base;
  int abort;
  // per-row metadata of the group
  int row_pos[BM];
  int row_slot[BM];
  int row_page[BM];       // -1: row has bad metadata
  int row_view[BM];
  int row_q[BM];          // row of q in shared memory (sequences padded to 16 rows)
  int row_seq[BM];        // sequence (index into sq_*) of each row
  // sequences of the group that have rows (each takes >= 16 padded q rows)
  int nseq;
  int sq_b[MAX_SEQ], sq_n[MAX_SEQ], sq_L[MAX_SEQ], sq_gr0[MAX_SEQ], sq_qoff[MAX_SEQ];
  int sq_npages[MAX_SEQ], sq_pg0[MAX_SEQ], sq_x0[MAX_SEQ], sq_nx[MAX_SEQ], sq_any[MAX_SEQ];
  int xs_slot[BM];        // per sequence: slots written by its view rows, ascending
  int xs_row[BM];         //   and the group rows that write them
  uint32_t xs_mask[BM][4];  //   and the rows of the sequence that see each of them
                            //   (bit j of word w: row 32 w + j)
  short pg_log[MAX_PAGES];  // per sequence: logical pages attended, in order
  int pg_phys[MAX_PAGES];   //   and their physical pages (-1: bad table entry)
  alignas(16) float lse2[BM];   // log2-sum-exp2 of the scaled scores of each row (float4 loads)
  float pm2[2][BM], pl2[2][BM];  // pass-1 partial (max, sum) per TMEM lane and warp half
  alignas(16) float red[4][BM];  // resident scores: per-quadrant row partials
  alignas(16) float row_m[BM];   //   row maximum (scaled, log2 domain; float4 loads)
  alignas(16) float row_inv[BM]; //   1 / row sum of exponentials (float4 loads)
};
static_assert(offsetof(Ctrl, lse2) % 16 == 0, "lse2 is read as float4");
static_assert(offsetof(Ctrl, row_m) % 16 == 0 && offsetof(Ctrl, row_inv) % 16 == 0,
              "row_m and row_inv are read as float4");
static_assert(sizeof(Ctrl) % 16 == 0 || true, "");
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

__device__ __forceinline__ bool aborted(Ctrl* c) {
  return *reinterpret_cast<volatile int*>(&c->abort) != 0;
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

// double -> float with round-to-odd: truncate toward zero, then set the
// last bit when the value was not exact. Rounding that float to bf16 to
// nearest even then gives the bf16 nearest to the double (Boldo and
// Melquiond, "When double rounding is odd"), i.e. a single rounding.
__device__ __forceinline__ float to_float_odd(double x) {
  const float f = __double2float_rz(x);
  const uint32_t odd = (double)f != x ? 1u : 0u;
  return __uint_as_float(__float_as_uint(f) | odd);
}

// Rotate-half RoPE of dimensions [32c, 32c + 32) and [64 + 32c, ...) in
// double from double cos / sin tables; the results come back as
// round-to-odd floats for the bf16 rounding that follows.
__device__ __forceinline__ void rope32(float* lo, float* hi, int pos, int c, const double* cos_t,
                                       const double* sin_t) {
  const double2* cp = reinterpret_cast<const double2*>(cos_t + (size_t)pos * (D / 2) + 32 * c);
  const double2* sp = reinterpret_cast<const double2*>(sin_t + (size_t)pos * (D / 2) + 32 * c);
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const double2 cs = __ldg(cp + u), sn = __ldg(sp + u);
    const double cv[2] = {cs.x, cs.y}, sv[2] = {sn.x, sn.y};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = 2 * u + e;
      const double a = lo[t], b = hi[t];
      lo[t] = to_float_odd(fma(a, cv[e], -b * sv[e]));
      hi[t] = to_float_odd(fma(b, cv[e], a * sv[e]));
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
                                      const double* cos_t, const double* sin_t, uint8_t* q,
                                      int c0 = 0, int c1 = 2) {
#pragma unroll 1
  for (int c = c0; c < c1; ++c) {
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
// Pass c covers dimensions [32c, 32c + 32) and [64 + 32c, 64 + 32c + 32)
// (the rotate-half pairs); passes [c0, c1) are done.
__device__ __forceinline__ void epi_kv(uint32_t taddr, int row, bool valid, bool rotate, int pos,
                                       const double* cos_t, const double* sin_t, uint8_t* dst,
                                       int c0 = 0, int c1 = 2) {
#pragma unroll 1
  for (int c = c0; c < c1; ++c) {
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

// q and k of dimensions [32c, 32c + 32) and their rotate-half partners
// [64 + 32c, ...) of this lane's row, in two sub-passes of 16 pairs: each
// cos / sin value is loaded once for both q and k. The rotation is the one
// of rope32 (double, round-to-odd), so the results are the same bits.
__device__ __forceinline__ void epi_qk(uint32_t trow, int c, int qrow, int row, bool valid, int pos,
                                       const double* cos_t, const double* sin_t, uint8_t* q,
                                       uint8_t* kst) {
#pragma unroll 1
  for (int s = 0; s < 2; ++s) {
    const int d0 = 32 * c + 16 * s;            // first (lo) dimension of the sub-pass
    float qlo[16], qhi[16], klo[16], khi[16];
    ptx::tmem_ld16(trow + d0, qlo);
    ptx::tmem_ld16(trow + 64 + d0, qhi);
    ptx::tmem_ld16(trow + 128 + d0, klo);
    ptx::tmem_ld16(trow + 192 + d0, khi);
    ptx::tmem_ld_wait();
    if (!valid) continue;
    const double2* cp = reinterpret_cast<const double2*>(cos_t + (size_t)pos * (D / 2) + d0);
    const double2* sp = reinterpret_cast<const double2*>(sin_t + (size_t)pos * (D / 2) + d0);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const double2 cs = __ldg(cp + u), sn = __ldg(sp + u);
      const double cv[2] = {cs.x, cs.y}, sv[2] = {sn.x, sn.y};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = 2 * u + e;
        const double a = qlo[t], b = qhi[t];
        qlo[t] = to_float_odd(fma(a, cv[e], -b * sv[e]));
        qhi[t] = to_float_odd(fma(b, cv[e], a * sv[e]));
        const double ka = klo[t], kb = khi[t];
        klo[t] = to_float_odd(fma(ka, cv[e], -kb * sv[e]));
        khi[t] = to_float_odd(fma(kb, cv[e], ka * sv[e]));
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int ch = d0 / 8 + u;               // 16-byte chunk of the d-half
      *reinterpret_cast<uint4*>(q + sw128(qrow, ch)) = pack8(qlo + 8 * u);
      *reinterpret_cast<uint4*>(q + HALF_BYTES + sw128(qrow, ch)) = pack8(qhi + 8 * u);
      *reinterpret_cast<uint4*>(kst + swz256(row, ch)) = pack8(klo + 8 * u);
      *reinterpret_cast<uint4*>(kst + swz256(row, 8 + ch)) = pack8(khi + 8 * u);
    }
  }
}

// Running log2-domain max m and sum l of one row over NK more scores v
// (raw S values; the scale sl2 = log2(e)/sqrt(D) is applied in the
// exponent's FMA). Keys whose bit in mk is clear are dropped before
// anything else, so a NaN in an unattended slot never reaches the sums.
// Eight independent max / sum chains.
template <int NK>
__device__ __forceinline__ void lse_block(float* v, uint64_t mk, float sl2, float& m, float& l) {
  float b8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) b8[i] = -INFINITY;
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    v[j] = ((mk >> j) & 1ull) ? v[j] : -INFINITY;
    b8[j & 7] = fmaxf(b8[j & 7], v[j]);
  }
  // rounding is monotone, so the scaled maximum is the maximum scaled score
  const float bm = fmaxf(fmaxf(fmaxf(b8[0], b8[1]), fmaxf(b8[2], b8[3])),
                         fmaxf(fmaxf(b8[4], b8[5]), fmaxf(b8[6], b8[7])));
  const float mn = fmaxf(m, bm * sl2);
  if (mn == -INFINITY) return;
  float s8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) s8[i] = 0.f;
#pragma unroll
  for (int j = 0; j < NK; ++j) s8[j & 7] += ptx::ex2(fmaf(v[j], sl2, -mn));
  l = l * ptx::ex2(m - mn) +
      (((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7])));
  m = mn;
}

// Reduction over the 32 lanes (keys) of a warp of NR row values per lane
// (NR = 8, 16 or 32): recursive halving, so that after log2(NR) exchange
// steps each lane holds one row, then plain butterflies over the lanes that
// share it. Returns the reduced value of row (lane >> (5 - log2 NR)).
template <int NR, bool kMax>
__device__ __forceinline__ float lane_reduce_rows(float (&v)[32], int lane) {
  constexpr int K = NR == 32 ? 5 : NR == 16 ? 4 : 3;
  static_assert(NR == 8 || NR == 16 || NR == 32, "rows per half");
#pragma unroll
  for (int step = 0; step < K; ++step) {
    const int off = 16 >> step;
    const int n = NR >> (step + 1);   // values kept after this step
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < n; ++i) {
      const float send = upper ? v[i] : v[i + n];
      const float keep = upper ? v[i + n] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, off);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  float r = v[0];
#pragma unroll
  for (int off = (16 >> K); off >= 1; off >>= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, r, off);
    r = kMax ? fmaxf(r, o) : r + o;
  }
  return r;
}

template <int NR>
__device__ __forceinline__ void tmem_ld_rows(uint32_t taddr, float* v) {
  if constexpr (NR == 32) ptx::tmem_ld32(taddr, v);
  else if constexpr (NR == 16) ptx::tmem_ld16(taddr, v);
  else ptx::tmem_ld8(taddr, v);
}

template <int NR>
__device__ __forceinline__ void tmem_st_rows(uint32_t taddr, const float* v) {
  if constexpr (NR == 32) ptx::tmem_st32(taddr, v);
  else if constexpr (NR == 16) ptx::tmem_st16(taddr, v);
  else ptx::tmem_st8(taddr, v);
}

// A sequence keeps all of its scores in TMEM (one S^T product per chunk,
// N16 columns each, O^T hi and lo later in the first two chunks' columns,
// or the unused columns after a single chunk) when its padded
// rows are a power of two up to 64 and its chunks fit the 512 columns.
__device__ __forceinline__ bool resident_fits(int N16, int nch) {
  return (N16 == 16 || N16 == 32 || N16 == 64) && nch >= 1 && nch * N16 <= 512;
}

// Schedule parameter of the one-tile kernel: none.
struct NoSched {
  int n_bins;
};

// kPersist: a persistent CTA runs the tiles of its schedule bin; otherwise
// CTA i runs tile i.
// kSplit (few tiles): a cluster of 4 CTAs per tile splits the projection's
// K range in four (each CTA streams a quarter of the head's Wqkv slice and
// issues a quarter of the products). After a cluster barrier every rank
// sends the fp32 partials of the blocks it does not own to their owners'
// shared memory (q: rank 0, k: rank 1, v: rank 2); after a second barrier
// each owner adds them to its own partial in TMEM, in rank order. The k and
// v owners write their rows to the cache and arrive on rank 0's kv_ready
// barrier; rank 0 keeps q on chip, waits for kv_ready (bounded) and runs
// the attention. Both cluster barriers are reached by every thread of every
// rank on every path (all other waits are bounded), and no CTA reads or
// writes another's shared memory after the second one except for those
// two arrivals on rank 0, which waits for them before it goes on.
template <bool kPersist, bool kSplit>
__global__ void __launch_bounds__(NTHREADS, 1)
    step_bf16_kernel(const __grid_constant__ StepPlan plan,
                     const __grid_constant__ std::conditional_t<kPersist, TileSched, NoSched> sched,
                     const __grid_constant__ StepArgs a,
                     const __grid_constant__ CUtensorMap tmap_x16,
                     const __grid_constant__ CUtensorMap tmap_x32,
                     const __grid_constant__ CUtensorMap tmap_x64,
                     const __grid_constant__ CUtensorMap tmap_x128,
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
  const int H = a.hidden;
  const int nkb = H / BK;
  constexpr int kStages = STAGES;
  constexpr int kStageBytes = STAGE_BYTES;
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
      ptx::mbar_init(&ctrl->s_empty[s], 8);
    }
    ptx::mbar_init(&ctrl->mma_done, 1);
    ptx::mbar_init(&ctrl->p_full, 8);
    ptx::mbar_init(&ctrl->pv_done, 1);
    ptx::mbar_init(&ctrl->q_ready, 8);
    ptx::mbar_init(&ctrl->o_done, 1);
    ptx::mbar_init(&ctrl->s_half, 1);
    ptx::mbar_init(&ctrl->s_all, 1);
    ptx::mbar_init(&ctrl->t_free, 8);
    ptx::mbar_init(&ctrl->pv_buf[0], 1);
    ptx::mbar_init(&ctrl->pv_buf[1], 1);
    ptx::mbar_init(&ctrl->p_buf[0], 8);
    ptx::mbar_init(&ctrl->p_buf[1], 8);
    ptx::mbar_init(&ctrl->kv_ready, 2);
    ctrl->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(&ctrl->tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 1) {
    ptx::prefetch_tmap(&tmap_x16);
    ptx::prefetch_tmap(&tmap_x32);
    ptx::prefetch_tmap(&tmap_x64);
    ptx::prefetch_tmap(&tmap_x128);
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_k);
    ptx::prefetch_tmap(&tmap_v);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;

  // Tiles of this CTA (a persistent CTA runs several, one after another;
  // barrier phases, schedule counters and TMEM carry over between them).
  int t_beg = 0, t_end = 1;
  // role (the rank in a split tile's cluster): 0 = q and attention
  // (everything when not split), 1 = k, 2 = v, 3 = a partial only; the
  // rank's quarter of the projection K steps is [kb0, kb1)
  int role = 0;
  int tile_id = (int)blockIdx.x;
  int kb0 = 0, kb1 = nkb;
  if constexpr (kSplit) {
    role = (int)ptx::cluster_ctarank();
    tile_id = (int)blockIdx.x / CL_RANKS;
    kb0 = role * (nkb / CL_RANKS);
    kb1 = kb0 + nkb / CL_RANKS;
  }
  if constexpr (kPersist) {
    t_beg = sched.bin0[blockIdx.x];
    t_end = sched.bin0[blockIdx.x + 1];
  }
  uint32_t kstep0 = 0;   // projection K steps of the earlier tiles
  // attention schedule counters, identical in every thread: chunk loads (K
  // or V) issued so far, S^T products, P.V products, finished sequences and
  // sequences whose q rows were repeated
  uint32_t ring = 0, scount = 0, ocount = 0, qcount = 0;
  // resident scores: sequences so far (s_half / s_all completions), P.V
  // chunks so far (P^T buffer (rp & 1), its barrier's use rp >> 1), and
  // t_free hand-overs. Each barrier completes at most once ahead of its
  // waiters, so its phase parity identifies the completion.
  uint32_t rcount = 0, rpcount = 0, tcount = 0;
  uint32_t opcount = 0;   // P.V chunks of two-pass sequences (p_full / pv_done completions)
  int64_t last_load = -1; // producer: the last attention chunk load actually issued
  for (int ti = t_beg; ti < t_end; ++ti) {
  int g, h;
  if constexpr (kPersist) {
    g = sched.tile[ti] >> 8;
    h = sched.tile[ti] & 255;
  } else {   // group-major numbering (groups in order of decreasing work)
    g = tile_id / a.n_heads;
    h = tile_id % a.n_heads;
  }
  // sequences of this group: plan.seq_order[seq_a .. seq_b); sequence b
  // owns q rows [seq_qoff[b], seq_qoff[b] + n_b) of the 128-row tile, which
  // are also the TMEM lanes of the projection
  const int seq_a = plan.group_seq0[g];
  const int seq_b = plan.group_seq0[g + 1];

  // ================================================================ projection
  if (warp == kProducerWarp) {
    if (lane == 0) {   // TMA producer
      // x boxes of the tile, computed once: each sequence's (16-padded) rows
      // in the largest boxes that fit (at most 8 boxes for 128 rows)
      int nbox = 0, x_rows = 0;
      uint32_t box_dst[8];
      int box_row[8], box_h[8];
      for (int q = seq_a; q < seq_b; ++q) {
        const int b = plan.seq_order[q];
        int rem = (plan.cu_rows[b + 1] - plan.cu_rows[b] + 15) & ~15;
        int off = 0;
        x_rows += rem;
        while (rem > 0 && nbox < 8) {
          const int hgt = rem >= 128 ? 128 : rem >= 64 ? 64 : rem >= 32 ? 32 : 16;
          box_dst[nbox] = (uint32_t)(plan.seq_qoff[b] + off) * 128u;
          box_row[nbox] = plan.cu_rows[b] + off;
          box_h[nbox] = hgt;
          ++nbox;
          off += hgt;
          rem -= hgt;
        }
      }
      // x rows are read by every head's tile of the group and a head's
      // Wqkv slice by every group's tile: keep both in L2
      const uint64_t pol_keep = ptx::policy_evict_last();
      int kissued = kb0;
      for (int kb = kb0; kb < kb1; ++kb) {
        const uint32_t kg = kstep0 + (kb - kb0);
        const int s = kg % kStages;
        const uint32_t u = kg / kStages;
        if (u > 0 && !wait_bar(ctrl, &ctrl->empty[s], (u - 1) & 1, a.err, 1)) break;
        if (u == 0 && aborted(ctrl)) break;
        kissued = kb + 1;
        uint8_t* st = smem + s * kStageBytes;
        ptx::mbar_arrive_expect_tx(&ctrl->full[s], B_BYTES + x_rows * BK * 2);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (i < nbox) {
            const CUtensorMap* mx = box_h[i] == 128 ? &tmap_x128 : box_h[i] == 64 ? &tmap_x64
                                  : box_h[i] == 32 ? &tmap_x32 : &tmap_x16;
            ptx::tma_load_2d_hint(st + box_dst[i], mx, kb * BK, box_row[i], &ctrl->full[s],
                                  pol_keep);
          }
        }
        // this head's q, k and v column blocks of Wqkv, two 64-column halves
        // each: one 48 KB box of the 5-D view (column, K row, half, block,
        // head), laid out as six [64 K rows][64 columns] sub-boxes
        ptx::tma_load_5d_hint(st + A_BYTES, &tmap_w, 0, kb * BK, 0, 0, h, &ctrl->full[s],
                              pol_keep);
      }
      // after a timeout: the stages still in flight land before this CTA
      // moves on (every earlier stage was consumed by a product that waited
      // for it)
      if (aborted(ctrl)) {
        for (int kb = kissued - kStages > kb0 ? kissued - kStages : kb0; kb < kissued; ++kb) {
          const uint32_t kg = kstep0 + (kb - kb0);
          ptx::mbar_wait(&ctrl->full[kg % kStages], (kg / kStages) & 1, WAIT_NS);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {   // MMA issuer
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(BM, 128, false, true);
      constexpr uint32_t idesc256 = ptx::idesc_bf16_f32(BM, 256, false, true);
      for (int kb = kb0; kb < kb1; ++kb) {
        const uint32_t kg = kstep0 + (kb - kb0);
        const int s = kg % kStages;
        const uint32_t u = kg / kStages;
        if (!wait_bar(ctrl, &ctrl->full[s], u & 1, a.err, 2)) break;
        ptx::tc_fence_after();
        const uint32_t a_base = ptx::smem_u32(smem + s * kStageBytes);
        const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          // A: K-major rows of 128 bytes; 8-row atoms 1024 bytes apart.
          const uint64_t ad = ptx::smem_desc_sw128(a_base + kk * 32, 16, 1024);
          // B: N-major (Wqkv rows are K); 64-column boxes 8 KB apart, 8-row
          // K groups 1024 bytes apart; K16 slice = 16 rows = 2 KB. q and k
          // (four boxes, 256 columns) go in one N=256 product, which reads
          // the A tile from shared memory once for both; v is N=128.
          const uint32_t acc = (kb != kb0 || kk != 0) ? 1u : 0u;
          const uint64_t bqk = ptx::smem_desc_sw128(b_base + kk * 2048, BOX_BYTES, 1024);
          ptx::umma_f16_ss(tmem, ad, bqk, idesc256, acc);
          const uint64_t bv = ptx::smem_desc_sw128(b_base + 4 * BOX_BYTES + kk * 2048,
                                                   BOX_BYTES, 1024);
          ptx::umma_f16_ss(tmem + 256, ad, bv, idesc, acc);
        }
        ptx::umma_commit(&ctrl->empty[s]);
      }
      ptx::umma_commit(&ctrl->mma_done);
    }
  } else {
    // ---- group metadata, built by warps 0..7 while the projection runs
    const int mt = tid;
    constexpr int NM = NSMX;
    if (mt == 0) {
      int ns = 0;
      for (int q = seq_a; q < seq_b; ++q) {
        const int b = plan.seq_order[q];
        const int n = plan.cu_rows[b + 1] - plan.cu_rows[b];
        if (n == 0 || ns >= MAX_SEQ) continue;
        ctrl->sq_b[ns] = b;
        ctrl->sq_n[ns] = n;
        ctrl->sq_L[ns] = plan.seq_lens[b];
        ctrl->sq_gr0[ns] = plan.cu_rows[b];
        ctrl->sq_qoff[ns] = plan.seq_qoff[b];
        ++ns;
      }
      ctrl->nseq = ns;
    }
    named_bar(2, NM);
    const int nseq = ctrl->nseq;
    // q rows of the tile: position, slot, page, view, sequence
    for (int i = mt; i < BM; i += NM) {
      int pos = 0, slot = 0, page = -1, view = 0, qr = i, sq = -1;
      for (int q = 0; q < nseq; ++q)
        if (i >= ctrl->sq_qoff[q] && i < ctrl->sq_qoff[q] + ctrl->sq_n[q]) sq = q;
      if (sq >= 0) {
        const int gr = ctrl->sq_gr0[sq] + (i - ctrl->sq_qoff[sq]);
        const int b = ctrl->sq_b[sq];
        pos = a.positions[gr];
        slot = a.slots ? a.slots[gr] : pos;
        view = a.view ? (int)a.view[gr] : 0;
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
      ctrl->row_seq[i] = sq;
    }
    named_bar(2, NM);
    // view rows with good metadata, per sequence
    if (mt < nseq) {
      int c = 0;
      for (int i = ctrl->sq_qoff[mt]; i < ctrl->sq_qoff[mt] + ctrl->sq_n[mt]; ++i)
        c += (ctrl->row_view[i] != 0 && ctrl->row_page[i] >= 0) ? 1 : 0;
      ctrl->sq_nx[mt] = c;
    }
    named_bar(2, NM);
    if (mt == 0) {
      int x = 0;
      for (int q = 0; q < nseq; ++q) {
        ctrl->sq_x0[q] = x;
        x += ctrl->sq_nx[q];
      }
    }
    named_bar(2, NM);
    // view slots of each sequence, ascending (rank sort)
    for (int i = mt; i < BM; i += NM) {
      if (ctrl->row_seq[i] < 0 || ctrl->row_view[i] == 0 || ctrl->row_page[i] < 0) continue;
      const int q = ctrl->row_seq[i];
      const int si = ctrl->row_slot[i];
      int rank = 0;
      for (int j = ctrl->sq_qoff[q]; j < ctrl->sq_qoff[q] + ctrl->sq_n[q]; ++j) {
        if (ctrl->row_view[j] == 0 || ctrl->row_page[j] < 0) continue;
        const int sj = ctrl->row_slot[j];
        rank += (sj < si || (sj == si && j < i)) ? 1 : 0;
      }
      ctrl->xs_slot[ctrl->sq_x0[q] + rank] = si;
      ctrl->xs_row[ctrl->sq_x0[q] + rank] = i;
    }
    named_bar(2, NM);
    // Flash-Verify visibility of each view slot, once per tile: row rr of
    // its sequence sees the slot written by row xr when both are of the
    // same view and rr's position is not before xr's
    {
      const int nxs = nseq > 0 ? ctrl->sq_x0[nseq - 1] + ctrl->sq_nx[nseq - 1] : 0;
      for (int it = mt; it < nxs * 4; it += NM) {
        const int x = it >> 2, w = it & 3;
        int q = 0;
        while (q + 1 < nseq && ctrl->sq_x0[q + 1] <= x) ++q;
        const int xr = ctrl->xs_row[x];
        const int kv = ctrl->row_view[xr], kp = ctrl->row_pos[xr];
        uint32_t m = 0u;
        for (int j = 0; j < 32; ++j) {
          const int col = 32 * w + j;
          if (col < ctrl->sq_n[q]) {
            const int rr = ctrl->sq_qoff[q] + col;
            if (ctrl->row_view[rr] == kv && ctrl->row_pos[rr] >= kp) m |= 1u << j;
          }
        }
        ctrl->xs_mask[x][w] = m;
      }
    }
    named_bar(2, NM);
    // logical pages: the context pages, then the pages of view slots past them
    if (mt < nseq) {
      const int npr = (ctrl->sq_L[mt] + PS - 1) / PS;
      int np = npr, last = -1;
      for (int t = 0; t < ctrl->sq_nx[mt]; ++t) {
        const int p = ctrl->xs_slot[ctrl->sq_x0[mt] + t] / PS;
        if (p >= npr && p != last) {
          ++np;
          last = p;
        }
      }
      ctrl->sq_npages[mt] = np;
    }
    named_bar(2, NM);
    if (mt == 0) {
      int o = 0;
      for (int q = 0; q < nseq; ++q) {
        ctrl->sq_pg0[q] = o;
        if (o + ctrl->sq_npages[q] > MAX_PAGES) {
          set_err(a.err, kDevBadSlot, -2);
          ctrl->sq_npages[q] = MAX_PAGES - o;
        }
        o += ctrl->sq_npages[q];
      }
    }
    named_bar(2, NM);
    for (int q = 0; q < nseq; ++q) {
      const int npr = min((ctrl->sq_L[q] + PS - 1) / PS, ctrl->sq_npages[q]);
      const int* bt = a.block_table + (size_t)ctrl->sq_b[q] * plan.max_blocks;
      for (int i = mt; i < npr; i += NM) {
        const int pg = bt[i];
        const bool ok = pg >= 0 && pg < a.num_pages;
        if (!ok) set_err(a.err, kDevBadPage, -1 - i);
        ctrl->pg_log[ctrl->sq_pg0[q] + i] = (short)i;
        ctrl->pg_phys[ctrl->sq_pg0[q] + i] = ok ? pg : -1;
      }
    }
    if (mt < nseq) {
      const int q = mt;
      const int npr = (ctrl->sq_L[q] + PS - 1) / PS;
      const int* bt = a.block_table + (size_t)ctrl->sq_b[q] * plan.max_blocks;
      int np = npr, last = -1;
      for (int t = 0; t < ctrl->sq_nx[q] && np < ctrl->sq_npages[q]; ++t) {
        const int p = ctrl->xs_slot[ctrl->sq_x0[q] + t] / PS;
        if (p >= npr && p != last) {
          const int pg = bt[p];
          const bool ok = pg >= 0 && pg < a.num_pages;
          if (!ok) set_err(a.err, kDevBadPage, -1 - p);
          ctrl->pg_log[ctrl->sq_pg0[q] + np] = (short)p;
          ctrl->pg_phys[ctrl->sq_pg0[q] + np] = ok ? pg : -1;
          ++np;
          last = p;
        }
      }
    }
    named_bar(2, NM);
    if (mt < nseq) {
      int any = 0;
      for (int i = 0; i < ctrl->sq_npages[mt]; ++i) any |= ctrl->pg_phys[ctrl->sq_pg0[mt] + i] >= 0;
      ctrl->sq_any[mt] = any;
    }
    // mass partials: zero (the softmax warps accumulate into them)
    if (a.mass_part && role == 0) {
      for (int q = 0; q < nseq; ++q) {
        float4* part = reinterpret_cast<float4*>(
            a.mass_part + ((size_t)h * plan.batch + ctrl->sq_b[q]) * plan.row_stride);
        for (int j = mt; j < plan.row_stride / 4; j += NM) part[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
  __syncwarp();
  __syncthreads();   // row metadata visible; producer and MMA loops issued

  // ================================================================ epilogue
  const bool acc_ok = wait_bar(ctrl, &ctrl->mma_done, 0, a.err, 3);
  __syncwarp();
  ptx::tc_fence_after();
  if constexpr (kSplit) {
    // Every rank's partial is final and every rank's ring is idle, so the
    // partial slots (in the ring region) may be written. Each rank sends
    // the blocks it does not own; thread (quadrant, half) moves the 64
    // columns `half` of its row. Only the lane quadrants that hold the
    // group's rows travel.
    int lanes_used = 0;
    for (int q = seq_a; q < seq_b; ++q) {
      const int b = plan.seq_order[q];
      const int top = plan.seq_qoff[b] + ((plan.cu_rows[b + 1] - plan.cu_rows[b] + 15) & ~15);
      lanes_used = top > lanes_used ? top : lanes_used;
    }
    const int quads_used = (lanes_used + 31) >> 5;
    ptx::tc_fence_before();
    ptx::cluster_sync();
    ptx::tc_fence_after();
    if (warp < 8 && (warp & 3) < quads_used) {
      const int quad = warp & 3, hh = warp >> 2;
      const int row = quad * 32 + lane;
      const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
      const uint32_t sbase = ptx::smem_u32(smem);
      for (int b = 0; b < 3; ++b) {
        if (b == role) continue;
        const int slot = role < b ? role : role - 1;
        const uint32_t rbase = ptx::mapa_shared(sbase + (uint32_t)(slot * CL_SLOT_BYTES), (uint32_t)b);
#pragma unroll 1
        for (int j = 0; j < 2; ++j) {
          float v[32];
          ptx::tmem_ld32(trow + 128 * b + 64 * hh + 32 * j, v);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const int c4 = 16 * hh + 8 * j + i4;   // column quad of the block
            ptx::st_cluster_v4(rbase + (uint32_t)(c4 * 128 + row) * 16u, v[4 * i4],
                               v[4 * i4 + 1], v[4 * i4 + 2], v[4 * i4 + 3]);
          }
        }
      }
    }
    ptx::tc_fence_before();
    ptx::cluster_sync();   // the partials have landed
    ptx::tc_fence_after();
    if (warp < 8 && role < 3 && (warp & 3) < quads_used) {
      // the owner: its own partial plus the three received ones, in the
      // order of the senders' ranks, back into its TMEM columns
      const int quad = warp & 3, hh = warp >> 2;
      const int row = quad * 32 + lane;
      const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
        float v[32];
        const uint32_t col = trow + 128 * role + 64 * hh + 32 * j;
        ptx::tmem_ld32(col, v);
        ptx::tmem_ld_wait();
#pragma unroll 1
        for (int sl = 0; sl < 3; ++sl) {
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const int c4 = 16 * hh + 8 * j + i4;
            const float4 p4 = *reinterpret_cast<const float4*>(
                smem + sl * CL_SLOT_BYTES + (c4 * 128 + row) * 16);
            v[4 * i4] += p4.x;
            v[4 * i4 + 1] += p4.y;
            v[4 * i4 + 2] += p4.z;
            v[4 * i4 + 3] += p4.w;
          }
        }
        ptx::tmem_st32(col, v);
      }
      ptx::tmem_st_wait();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
  }
  {
    const int quad = warp & 3;
    const int i = quad * 32 + lane;
    const bool valid = acc_ok && ctrl->row_page[i] >= 0;
    const int pos = ctrl->row_pos[i];
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    // warps 0-3: q and the first v pass; warps 4-7: k and the second v
    // pass (v needs no rotation, so the halves balance)
    if (warp >= 8) {
      // producer and MMA warps take no part in the epilogue
    } else if (kSplit) {
      // the owner's block, warp half c taking dimensions [32c, 32c + 32)
      // and their rotate-half partners
      const int c = warp >> 2;
      if (role == 0)
        epi_q(trow + 0, ctrl->row_q[i], valid, pos, a.rope_cos, a.rope_sin, smem + Q_OFF, c, c + 1);
      else if (role == 1)
        epi_kv(trow + 128, i, valid, true, pos, a.rope_cos, a.rope_sin, smem + KST_OFF, c, c + 1);
      else if (role == 2)
        epi_kv(trow + 256, i, valid, false, pos, a.rope_cos, a.rope_sin, smem + VST_OFF, c, c + 1);
    } else {
      // warp half c: q and k of dimensions [32c, 32c + 32) (+ partners),
      // then the v pass c
      const int c = warp >> 2;
      epi_qk(trow, c, ctrl->row_q[i], i, valid, pos, a.rope_cos, a.rope_sin, smem + Q_OFF,
             smem + KST_OFF);
      epi_kv(trow + 256, i, valid, false, pos, a.rope_cos, a.rope_sin, smem + VST_OFF, c, c + 1);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();

  // Fresh k/v rows -> cache slots (16 consecutive threads per 256-byte row).
  {
    const size_t head_stride = (size_t)PS * D;
    __nv_bfloat16* kp = reinterpret_cast<__nv_bfloat16*>(a.k_pool);
    __nv_bfloat16* vp = reinterpret_cast<__nv_bfloat16*>(a.v_pool);
    for (int idx = tid; idx < BM * 32; idx += NTHREADS) {
      const int r = idx >> 5;
      const int part = idx & 31;
      const int ch = part & 15;
      if (kSplit && (role == 0 || role == 3 || (role == 1) != (part < 16))) continue;
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
  if constexpr (kSplit) {
    // k / v owners: every thread's cache stores, then one arrival (release,
    // cluster scope) on rank 0's kv_ready. A test can withhold the arrivals
    // (split_wait_epoch != split_epoch), so that rank 0's bounded wait runs
    // out.
    __threadfence();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if ((role == 1 || role == 2) && tid == 0 && a.split_wait_epoch == a.split_epoch)
      ptx::mbar_arrive_remote(ptx::mapa_shared(ptx::smem_u32(&ctrl->kv_ready), 0u));
    // rank 0: both arrivals (acquire), then the cache is read through TMA
    if (role == 0 && tid == 0) {
      if (!ptx::mbar_wait_cluster(&ctrl->kv_ready, 0, a.flag_wait_ns)) {
        set_err(a.err, kDevTimeout, 30);
        atomicExch(&ctrl->abort, 1);
      }
    }
    __syncthreads();
    asm volatile("fence.proxy.async.global;" ::: "memory");
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();

  // ================================================================ attention
  const float sl2 = 1.4426950408889634f * rsqrtf((float)D);   // log2(e) / sqrt(D)
  const uint32_t q_base = ptx::smem_u32(smem + Q_OFF);
  const uint32_t slot_base = ptx::smem_u32(smem + SLOT_OFF);
  const uint32_t pt_base = ptx::smem_u32(smem + PT_OFF);
  const uint32_t qrep_base = ptx::smem_u32(smem + QREP_OFF);

  // ranks 1-3 of a split tile stop here, and so does rank 0 when its wait
  // for the k / v owners gave up: it issues no load and no product, so
  // nothing is left in flight (its out rows stay unwritten, its mass
  // partials zero, and the error word holds the timeout)
  const bool gave_up = kSplit && *reinterpret_cast<volatile int*>(&ctrl->abort) != 0;
  const int nseq_g = (role == 0 && !gave_up) ? ctrl->nseq : 0;
  auto seq_resident = [&](int q) -> bool {
    const int n16 = (ctrl->sq_n[q] + 15) & ~15;
    return resident_fits(n16, (ctrl->sq_npages[q] + 1) >> 1);
  };
  for (int si = 0; si < nseq_g; ++si) {
    const int b = ctrl->sq_b[si];
    const int n = ctrl->sq_n[si];
    const int ra = ctrl->sq_qoff[si];           // first q row (row metadata index)
    const int gr0 = ctrl->sq_gr0[si];           // first row in x / out
    const int L = ctrl->sq_L[si];
    const int N16 = (n + 15) & ~15;
    const int qoff = ctrl->sq_qoff[si];
    const int npages = ctrl->sq_npages[si];
    const int nx = ctrl->sq_nx[si];
    const bool any_page = ctrl->sq_any[si] != 0;
    const short* pgl = ctrl->pg_log + ctrl->sq_pg0[si];
    const int* pgp = ctrl->pg_phys + ctrl->sq_pg0[si];
    const int* xsl = ctrl->xs_slot + ctrl->sq_x0[si];
    const int nch = (npages + 1) >> 1;
    // Resident scores (a sequence of 16, 32 or 64 padded rows whose chunks
    // fit TMEM): one S^T = K Q^T product per chunk into its own TMEM
    // columns, so K is read once; the softmax warps reduce the row maxima
    // and sums across lanes and form P from the same scores; O^T hi and lo
    // accumulate in the first two chunks' columns once both have been read.
    // Otherwise the two-pass scheme below. Where this sequence or the one
    // before it is resident, its first product waits until the softmax
    // warps have released the earlier sequence's TMEM (t_free).
    const bool res = resident_fits(N16, nch);
    const bool wait_free = si > 0 && (res || seq_resident(si - 1));
    const bool give_free = si + 1 < nseq_g && (res || seq_resident(si + 1));
    // Pass 1 keeps the rows on TMEM lanes. A sequence of at most 64 rows
    // is repeated R times (copy rho on lanes [rho*RS, rho*RS + N16)), so
    // that every lane quadrant (every SM sub-partition) holds rows; copy
    // rho takes the chunk's keys [rho*KR, rho*KR + KR), split between the
    // two warps of its quadrant. A wider sequence uses the group's q rows.
    const bool wide = N16 > 64;
    const int R = N16 <= 32 ? 4 : (N16 <= 64 ? 2 : 1);
    const int RS = 128 / R;
    const int KR = 128 / R;
    const uint32_t ptl_off = (uint32_t)N16 * 256u;   // P^T lo rows right after the hi rows
    float* part = a.mass_part ? a.mass_part + ((size_t)h * plan.batch + b) * plan.row_stride
                              : nullptr;
    // Chunk loads of this sequence, in ring order: pass 1 K_0 .. K_{nch-1}
    // (items r0 + c); pass 2 K_0, K_1, then V_c followed by K_{c+2}, so that
    // K runs one chunk ahead of V and each load's slot was freed by a
    // product issued a chunk earlier.
    const uint32_t r0 = ring, s0 = scount;
    const int npre = nch < 2 ? nch : 2;
    const int nk2 = nch > 2 ? nch - 2 : 0;
    auto item_v2 = [&](int c) -> uint32_t {
      return r0 + nch + npre + c + (c < nk2 ? c : nk2);
    };
    auto item_k2 = [&](int c) -> uint32_t { return c < 2 ? r0 + nch + c : item_v2(c - 2) + 1; };

    if (warp == kProducerWarp) {
      // ---------------------------------------- TMA producer
      if (lane == 0) {
        uint32_t item = r0;
        // pass-1 K chunks come back for pass 2 a few chunks later: keep
        // them in L2; pass-2 K and V are read for the last time
        const uint64_t pol_keep = ptx::policy_evict_last();
        const uint64_t pol_drop = ptx::policy_evict_first();
        auto load = [&](int c, bool is_v, uint64_t pol) {
          const int s = item % NSLOT;
          const uint32_t u = item / NSLOT;
          // after a timeout nothing more is issued (the slot may still be read)
          const bool free_ok = u > 0 ? wait_bar(ctrl, &ctrl->aempty[s], (u - 1) & 1, a.err, 10)
                                     : !aborted(ctrl);
          if (!free_ok) {
            ++item;
            return;
          }
          uint32_t bytes = 0;
          int phys[2] = {-1, -1};
          for (int pi = 0; pi < 2; ++pi) {
            const int pidx = 2 * c + pi;
            if (pidx < npages && pgp[pidx] >= 0) {
              phys[pi] = pgp[pidx];
              bytes += 2 * BOX_BYTES;
            }
          }
          ptx::mbar_arrive_expect_tx(&ctrl->afull[s], bytes);
          uint8_t* dst = smem + SLOT_OFF + s * SLOT_BYTES;
          const CUtensorMap* map = is_v ? &tmap_v : &tmap_k;
          for (int pi = 0; pi < 2; ++pi) {
            if (phys[pi] < 0) continue;
            const int row = ((layer * a.num_pages + phys[pi]) * a.n_heads + h) * PS;
            ptx::tma_load_2d_hint(dst + pi * BOX_BYTES, map, 0, row, &ctrl->afull[s], pol);
            ptx::tma_load_2d_hint(dst + HALF_BYTES + pi * BOX_BYTES, map, 64, row, &ctrl->afull[s],
                                  pol);
          }
          last_load = item;
          ++item;
        };
        if (res) {   // every chunk's K, then every chunk's V, each read once
          for (int c = 0; c < nch; ++c) load(c, false, pol_drop);
          for (int c = 0; c < nch; ++c) load(c, true, pol_drop);
        } else {
          for (int c = 0; c < nch; ++c) load(c, false, pol_keep);
          for (int c = 0; c < npre; ++c) load(c, false, pol_drop);
          for (int c = 0; c < nch; ++c) {
            load(c, true, pol_drop);
            if (c + 2 < nch) load(c + 2, false, pol_drop);
          }
        }
      }
    } else if (warp == kMmaWarp) {
      // ---------------------------------------- MMA issuer
      if (lane == 0 && wait_free) wait_bar(ctrl, &ctrl->t_free, (tcount - 1) & 1, a.err, 17);
      if (lane == 0 && res) {
        const uint32_t idesc_s = ptx::idesc_bf16_f32(128, N16, false, false);
        const uint32_t idesc_pv = ptx::idesc_bf16_f32(128, 2 * N16, true, true);
        // S^T_c = K_c Q^T into columns [c * N16, (c + 1) * N16)
        for (int c = 0; c < nch; ++c) {
          const uint32_t item = r0 + c;
          const int s = item % NSLOT;
          // after a timeout no product is issued
          if (wait_bar(ctrl, &ctrl->afull[s], (item / NSLOT) & 1, a.err, 11)) {
            ptx::tc_fence_after();
            const uint32_t kbase = slot_base + s * SLOT_BYTES;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
              const uint64_t kd = ptx::smem_desc_sw128(kbase + off, 16, 1024);
              const uint64_t qd = ptx::smem_desc_sw128(q_base + off + qoff * 128, 16, 1024);
              ptx::umma_f16_ss(tmem + (uint32_t)(c * N16), kd, qd, idesc_s, kk > 0 ? 1u : 0u);
            }
            ptx::umma_commit(&ctrl->aempty[s]);
          }
          if (c == (nch + 1) / 2 - 1) ptx::umma_commit(&ctrl->s_half);
        }
        ptx::umma_commit(&ctrl->s_all);
        // O^T += V_c^T P_c^T into columns [0, 2 N16): hi rows of P^T into
        // [0, N16), lo rows into [N16, 2 N16). Chunks 0 and 1 own those
        // columns, so the first product also waits for P_1 (its scores read).
        // P^T alternates between two buffers.
        bool any = false;
        for (int c = 0; c < nch; ++c) {
          const uint32_t vitem = r0 + nch + c;
          const int vs = vitem % NSLOT;
          const uint32_t rp = rpcount + (uint32_t)c;
          const uint32_t pbuf = pt_base + (rp & 1u) * 32768u;
          // per-buffer barriers: with two buffers the softmax warps can
          // publish P_{c+1} before this thread has seen P_c, and a single
          // barrier would then be two completions ahead of its waiter
          if (!wait_bar(ctrl, &ctrl->afull[vs], (vitem / NSLOT) & 1, a.err, 13) ||
              !wait_bar(ctrl, &ctrl->p_buf[rp & 1u], (rp >> 1) & 1, a.err, 14))
            continue;   // after a timeout no product is issued
          if (c == 0 && nch > 1 &&
              !wait_bar(ctrl, &ctrl->p_buf[(rp + 1) & 1u], ((rp + 1) >> 1) & 1, a.err, 14))
            continue;
          ptx::tc_fence_after();
          const uint32_t vbase = slot_base + vs * SLOT_BYTES;
          for (int pi = 0; pi < 2; ++pi) {
            const int pidx = 2 * c + pi;
            if (pidx >= npages || pgp[pidx] < 0) continue;
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const int ks = pi * 4 + k4;
              const uint64_t ad = ptx::smem_desc_sw128(vbase + ks * 2048, HALF_BYTES, 1024);
              const uint64_t bd = ptx::smem_desc_noswz(pbuf + ks * 256, 128, 2048);
              ptx::umma_f16_ss(tmem, ad, bd, idesc_pv, any ? 1u : 0u);
              any = true;
            }
          }
          ptx::umma_commit(&ctrl->aempty[vs]);
          ptx::umma_commit(&ctrl->pv_buf[rp & 1u]);
        }
        ptx::umma_commit(&ctrl->o_done);
      } else if (lane == 0) {
        const uint32_t idesc_std = ptx::idesc_bf16_f32(128, 128, false, false);
        const uint32_t idesc_s = ptx::idesc_bf16_f32(128, N16, false, false);
        const uint32_t idesc_pv = ptx::idesc_bf16_f32(128, 2 * N16, true, true);
        // Score product number j of this sequence from chunk-load `item`:
        // pass 1 S = Q K^T (rows of the whole group on lanes, keys on
        // columns), pass 2 S^T = K Q^T (keys on lanes, this sequence's rows
        // on columns).
        auto issue_s = [&](uint32_t j, uint32_t item, bool transposed) {
          const int s = item % NSLOT;
          const uint32_t idx = s0 + j;
          const uint32_t sb = idx & 1, su = idx >> 1;
          // after a timeout no product is issued
          if (!wait_bar(ctrl, &ctrl->afull[s], (item / NSLOT) & 1, a.err, 11)) return;
          if (su > 0 && !wait_bar(ctrl, &ctrl->s_empty[sb], (su - 1) & 1, a.err, 12)) return;
          ptx::tc_fence_after();
          const uint32_t kbase = slot_base + s * SLOT_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
            // K chunk and q rows, both K-major 128-byte swizzled.
            const uint64_t kd = ptx::smem_desc_sw128(kbase + off, 16, 1024);
            if (transposed) {
              const uint64_t qd = ptx::smem_desc_sw128(q_base + off + qoff * 128, 16, 1024);
              ptx::umma_f16_ss(tmem + (sb ? TM_S1 : TM_S0), kd, qd, idesc_s, kk > 0 ? 1u : 0u);
            } else {
              const uint64_t qd = ptx::smem_desc_sw128((wide ? q_base : qrep_base) + off, 16, 1024);
              ptx::umma_f16_ss(tmem + (sb ? TM_S1 : TM_S0), qd, kd, idesc_std, kk > 0 ? 1u : 0u);
            }
          }
          ptx::umma_commit(&ctrl->s_full[sb]);
          ptx::umma_commit(&ctrl->aempty[s]);
        };
        if (!wide) wait_bar(ctrl, &ctrl->q_ready, qcount & 1, a.err, 16);
        for (int c = 0; c < nch; ++c) issue_s(c, r0 + c, false);
        for (int c = 0; c < npre; ++c) issue_s(nch + c, item_k2(c), true);
        bool any = false;
        for (int c = 0; c < nch; ++c) {
          const uint32_t vitem = item_v2(c);
          const int vs = vitem % NSLOT;
          if (!wait_bar(ctrl, &ctrl->afull[vs], (vitem / NSLOT) & 1, a.err, 13) ||
              !wait_bar(ctrl, &ctrl->p_full, (opcount + c) & 1, a.err, 14))
            continue;   // after a timeout no product is issued
          ptx::tc_fence_after();
          const uint32_t vbase = slot_base + vs * SLOT_BYTES;
          for (int pi = 0; pi < 2; ++pi) {
            const int pidx = 2 * c + pi;
            if (pidx >= npages || pgp[pidx] < 0) continue;
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const int ks = pi * 4 + k4;   // 16 keys per step
              // A = V^T: M = d, N-major in shared memory (64 d per 128-byte
              // row), two 64-d blocks 16 KB apart (LBO), 8-key groups 1 KB
              // apart (SBO).
              const uint64_t ad = ptx::smem_desc_sw128(vbase + ks * 2048, HALF_BYTES, 1024);
              // B = P^T: N-major core matrices without swizzle: 8-key
              // groups 128 B apart (LBO), 8-row blocks 2048 B apart (SBO).
              const uint64_t bd = ptx::smem_desc_noswz(pt_base + ks * 256, 128, 2048);
              ptx::umma_f16_ss(tmem + TM_O, ad, bd, idesc_pv, any ? 1u : 0u);
              any = true;
            }
          }
          ptx::umma_commit(&ctrl->aempty[vs]);
          ptx::umma_commit(&ctrl->pv_done);
          if (c + 2 < nch) issue_s(nch + c + 2, item_k2(c + 2), true);
        }
        ptx::umma_commit(&ctrl->o_done);
      }
    } else {
      // ---------------------------------------- softmax warps 0-7
      // TMEM lane t (a q row in pass 1, a key in pass 2, a head dimension
      // for O^T) is shared by warps `quad` and `quad + 4`, which split the
      // columns between them (`half`).
      const int quad = warp & 3;
      const int half = warp >> 2;
      const int t = quad * 32 + lane;
      const uint32_t tl = (uint32_t)(quad * 32) << 16;
      // cat: 0 nobody attends the key, 1 every row does, 2 a view row's
      // slot (xi: its index among the sequence's view slots)
      auto key_info = [&](int c, int& slot, int& cat, int& xi) {
        const int pidx = 2 * c + (t >> 6);
        cat = 0;
        xi = -1;
        slot = -1;
        if (pidx >= npages || pgp[pidx] < 0) return;
        slot = (int)pgl[pidx] * PS + (t & 63);
        if (slot < L) {
          cat = 1;
          return;
        }
        int lo = 0, hi = nx - 1;
        while (lo <= hi) {
          const int mid = (lo + hi) >> 1;
          const int v = xsl[mid];
          if (v == slot) {
            cat = 2;
            xi = mid;
            return;
          }
          if (v < slot) lo = mid + 1; else hi = mid - 1;
        }
      };
      // Visibility of this thread's key to the 32 rows [32*blk, 32*blk+32)
      // of the sequence, as a bit mask.
      const uint32_t (*xsm)[4] = ctrl->xs_mask + ctrl->sq_x0[si];
      auto vis_mask = [&](int cat, int xi, int blk) -> uint32_t {
        if (cat == 0) return 0u;
        if (cat == 1) {
          const int lim = n - 32 * blk;
          return lim >= 32 ? 0xffffffffu : (lim <= 0 ? 0u : ((1u << lim) - 1u));
        }
        return xsm[xi][blk];
      };

      // ----- resident scores (see above). Thread t owns key t of every
      // chunk; the warp pair of a lane quadrant splits the rows in halves of
      // NR = N16 / 2 (warp half h: rows [h * NR, h * NR + NR)).
      auto resident_softmax = [&](auto nr_const) {
        constexpr int NR = decltype(nr_const)::value;
        constexpr int LPR = 32 / NR;                // lanes that share a reduced row
        const int rbase = half * NR;
        const uint32_t cbase = tmem + tl + (uint32_t)rbase;
        auto row_mask = [&](int c, int& slot, int& cat) -> uint32_t {
          int xi;
          key_info(c, slot, cat, xi);
          const uint32_t m = vis_mask(cat, xi, rbase >> 5) >> (rbase & 31);
          return NR == 32 ? m : (m & ((1u << NR) - 1u));
        };
        float acc[32];
        // sweep 1: row maxima of the raw scores, this thread's keys (the
        // first half of the chunks as soon as their products land), then
        // across the lanes and the four quadrants
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = -INFINITY;
        for (int c = 0; c < nch; ++c) {
          int slot, cat;
          const uint32_t mk = row_mask(c, slot, cat);
          if (c == 0 || c == (nch + 1) / 2) {
            wait_bar(ctrl, c == 0 ? &ctrl->s_half : &ctrl->s_all, rcount & 1, a.err, 25);
            ptx::tc_fence_after();
          }
          float v[32];
          tmem_ld_rows<NR>(cbase + (uint32_t)(c * N16), v);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < NR; ++j)
            if ((mk >> j) & 1u) acc[j] = fmaxf(acc[j], v[j]);
        }
        {
          const float r = lane_reduce_rows<NR, true>(acc, lane);
          if ((lane & (LPR - 1)) == 0) ctrl->red[quad][rbase + lane / LPR] = r;
        }
        named_bar(1, NSMX);
        for (int rr = tid; rr < N16; rr += NSMX) {
          const float m = fmaxf(fmaxf(ctrl->red[0][rr], ctrl->red[1][rr]),
                                fmaxf(ctrl->red[2][rr], ctrl->red[3][rr]));
          // rounding is monotone, so the scaled maximum is the maximum scaled score
          ctrl->row_m[rr] = m * sl2;
        }
        named_bar(1, NSMX);
        // sweep 2: e = 2^(s * sl2 - m) (0 where the key is not visible),
        // summed per row, and stored back over the scores for sweep 3
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = 0.f;
        for (int c = 0; c < nch; ++c) {
          int slot, cat;
          const uint32_t mk = row_mask(c, slot, cat);
          float v[32];
          tmem_ld_rows<NR>(cbase + (uint32_t)(c * N16), v);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j4 = 0; j4 < NR; j4 += 4) {
            const float4 m4 = *reinterpret_cast<const float4*>(ctrl->row_m + rbase + j4);
            const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = j4 + e;
              v[j] = ((mk >> j) & 1u) ? ptx::ex2(fmaf(v[j], sl2, -mm[e])) : 0.f;
              acc[j] += v[j];
            }
          }
          tmem_st_rows<NR>(cbase + (uint32_t)(c * N16), v);
        }
        ptx::tmem_st_wait();
        {
          const float r = lane_reduce_rows<NR, false>(acc, lane);
          if ((lane & (LPR - 1)) == 0) ctrl->red[quad][rbase + lane / LPR] = r;
        }
        named_bar(1, NSMX);
        for (int rr = tid; rr < N16; rr += NSMX) {
          const float l = (ctrl->red[0][rr] + ctrl->red[1][rr]) + (ctrl->red[2][rr] + ctrl->red[3][rr]);
          ctrl->row_inv[rr] = l > 0.f ? 1.f / l : 0.f;
        }
        named_bar(1, NSMX);
        // sweep 3, chunk by chunk: P = e / l, the per-key mass, P^T (bf16 hi
        // + lo) for the P.V product, in two buffers that alternate
        for (int c = 0; c < nch; ++c) {
          int slot, cat;
          (void)row_mask(c, slot, cat);
          const int pidx = 2 * c + (t >> 6);
          const bool loaded = pidx < npages && pgp[pidx] >= 0;
          const uint32_t rp = rpcount + (uint32_t)c;
          uint8_t* pth = smem + PT_OFF + (rp & 1u) * 32768u;
          uint8_t* ptl = pth + ptl_off;
          float v[32];
          tmem_ld_rows<NR>(cbase + (uint32_t)(c * N16), v);
          ptx::tmem_ld_wait();
          // this chunk's scores are read (chunks 0 and 1 take O^T next)
          ptx::tc_fence_before();
          // this P^T buffer is free once the product two chunks back
          // completed; P^T is then written eight rows at a time
          if (rp >= 2) wait_bar(ctrl, &ctrl->pv_buf[rp & 1u], ((rp >> 1) - 1) & 1, a.err, 23);
          float msum = 0.f;
#pragma unroll
          for (int g8 = 0; g8 < NR / 8; ++g8) {
            uint32_t ph[4], pq[4];
#pragma unroll
            for (int j4 = 0; j4 < 8; j4 += 4) {
              const int j = 8 * g8 + j4;
              const float4 i4 = *reinterpret_cast<const float4*>(ctrl->row_inv + rbase + j);
              const float p0 = v[j] * i4.x, p1 = v[j + 1] * i4.y;
              const float p2 = v[j + 2] * i4.z, p3 = v[j + 3] * i4.w;
              msum += (p0 + p1) + (p2 + p3);
              ptx::split_bf16(p0, p1, ph[j4 >> 1], pq[j4 >> 1]);
              ptx::split_bf16(p2, p3, ph[(j4 >> 1) + 1], pq[(j4 >> 1) + 1]);
            }
            const int nb = (rbase >> 3) + g8;      // 8-row block of the sequence
            *reinterpret_cast<uint4*>(pth + nb * 2048 + t * 16) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
            *reinterpret_cast<uint4*>(ptl + nb * 2048 + t * 16) = make_uint4(pq[0], pq[1], pq[2], pq[3]);
          }
          // both halves add into the zeroed mass row: two addends, so the
          // result does not depend on their order
          if (part && cat != 0) atomicAdd(part + slot, msum);
          const uint32_t vitem = r0 + nch + c;
          const int vs = vitem % NSLOT;
          if (loaded && cat == 0) {
            // V rows of keys nobody attends may hold anything: zero them
            wait_bar(ctrl, &ctrl->afull[vs], (vitem / NSLOT) & 1, a.err, 22);
            uint8_t* vrow = smem + SLOT_OFF + vs * SLOT_BYTES + half * HALF_BYTES +
                            (t >> 6) * BOX_BYTES + (t & 63) * 128;
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(vrow + ch * 16) = z;
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&ctrl->p_buf[rp & 1u]);
        }
      };
      if (res) {
        if (N16 == 16)
          resident_softmax(std::integral_constant<int, 8>{});
        else if (N16 == 32)
          resident_softmax(std::integral_constant<int, 16>{});
        else
          resident_softmax(std::integral_constant<int, 32>{});
      } else {

      // ----- repeated q rows for pass 1 (sequences of at most 64 rows):
      // lane t holds row t % RS. A 128-byte row's swizzle phase depends on
      // its index mod 8, which the copy preserves, so rows copy verbatim.
      if (!wide) {
        for (int i = tid; i < 128 * 16; i += NSMX) {
          const int lt = i >> 4;
          const int hd = (i >> 3) & 1;
          const int c8 = i & 7;
          const int r = lt % RS;
          if (r >= N16) continue;
          const uint4 v = *reinterpret_cast<const uint4*>(smem + Q_OFF + hd * HALF_BYTES +
                                                          (qoff + r) * 128 + c8 * 16);
          *reinterpret_cast<uint4*>(smem + QREP_OFF + hd * HALF_BYTES + lt * 128 + c8 * 16) = v;
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&ctrl->q_ready);
      }

      // ----- pass 1: log-sum-exp of every row. S = Q K^T has rows on TMEM
      // lanes: thread t owns one row copy and half of the copy's keys of
      // every chunk (KR / 2 of them), keeping a running max and sum; the
      // partial pairs of all copies and both halves are merged at the end.
      {
        const int rho = wide ? 0 : t / RS;
        const int r = wide ? t - qoff : t - rho * RS;   // sequence row of lane t
        const bool active = r >= 0 && r < n;
        const bool warp_active = __any_sync(0xffffffffu, active);
        const int myview = active ? ctrl->row_view[ra + r] : 0;
        const int KH = KR >> 1;                      // keys per thread per chunk
        const int jbeg = rho * KR + half * KH;       // first chunk column of this thread
        float m = -INFINITY, l = 0.f;
        for (int c = 0; c < nch; ++c) {
          const uint32_t idx = s0 + c;
          const uint32_t sb = idx & 1;
          // This thread's keys [jbeg, jbeg + KH) of the chunk lie in one
          // page, pidx (KH = 64, 32 or 16 and jbeg a multiple of KH); its
          // row attends the page's context slots, then view slots of its
          // own view at positions <= its own. The mask is formed before
          // the scores are waited for.
          uint64_t km = 0ull;
          if (warp_active) {
            const int pidx = 2 * c + (jbeg >> 6);
            if (active && pidx < npages && pgp[pidx] >= 0) {
              const int plog = (int)pgl[pidx];
              const int nv = min(max(L - plog * PS, 0), PS);
              km = nv >= 64 ? ~0ull : ((1ull << nv) - 1ull);
              if (nv < PS && myview != 0) {
                for (int x = 0; x < nx; ++x) {
                  const int xs = xsl[x];
                  if (xs / PS == plog && ((xsm[x][r >> 5] >> (r & 31)) & 1u))
                    km |= 1ull << (xs % PS);
                }
              }
              km >>= (jbeg & 63);
            }
          }
          wait_bar(ctrl, &ctrl->s_full[sb], (idx >> 1) & 1, a.err, 20);
          ptx::tc_fence_after();
          if (warp_active) {
            const uint32_t sbase = tmem + tl + (sb ? TM_S1 : TM_S0) + jbeg;
            if (KH == 64) {
              // both loads in flight before the one wait
              float v[64];
              ptx::tmem_ld32(sbase, v);
              ptx::tmem_ld32(sbase + 32, v + 32);
              ptx::tmem_ld_wait();
              lse_block<64>(v, km, sl2, m, l);
            } else if (KH == 32) {
              float v[32];
              ptx::tmem_ld32(sbase, v);
              ptx::tmem_ld_wait();
              lse_block<32>(v, km, sl2, m, l);
            } else {
              float v[16];
              ptx::tmem_ld16(sbase, v);
              ptx::tmem_ld_wait();
              lse_block<16>(v, km, sl2, m, l);
            }
          }
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&ctrl->s_empty[sb]);
        }
        ctrl->pm2[half][t] = m;
        ctrl->pl2[half][t] = l;
        named_bar(1, NSMX);
        for (int rr = tid; rr < n; rr += NSMX) {
          float M = -INFINITY;
          for (int q = 0; q < R; ++q)
            for (int hp = 0; hp < 2; ++hp)
              M = fmaxf(M, ctrl->pm2[hp][wide ? qoff + rr : q * RS + rr]);
          float S = 0.f;
          if (M != -INFINITY) {
            for (int q = 0; q < R; ++q)
              for (int hp = 0; hp < 2; ++hp) {
                const int lt = wide ? qoff + rr : q * RS + rr;
                const float mq = ctrl->pm2[hp][lt];
                if (mq != -INFINITY) S += ctrl->pl2[hp][lt] * ptx::ex2(mq - M);
              }
          }
          ctrl->lse2[rr] = S > 0.f ? M + log2f(S) : INFINITY;
        }
        named_bar(1, NSMX);
      }

      // ----- pass 2: probabilities, mass, P^T for the P.V product. S^T has
      // the chunk's keys on TMEM lanes (thread t owns key t) and this
      // sequence's rows on columns; warp half `half` takes the NC = N16 / 2
      // rows [half * NC, half * NC + NC). Its scores are loaded (at most two
      // 32-column loads in flight) while the previous chunk's P.V product
      // may still be reading the single P^T buffer; once both are done the
      // TMEM buffer is released and P^T is written eight rows at a time.
      const int NC = N16 >> 1;
      const int c0 = half * NC;
      // visibility of this thread's key to the rows [c0, c0 + 64), bit j for row c0 + j
      auto vis_bits = [&](int cat, int xi) -> uint64_t {
        if (cat == 0) return 0ull;
        const int lim = n - c0;
        if (cat == 1) return lim >= 64 ? ~0ull : (lim <= 0 ? 0ull : ((1ull << lim) - 1ull));
        const int w = c0 >> 5, sh = c0 & 31;
        const uint64_t lo = (uint64_t)xsm[xi][w] | ((w + 1 < 4 ? (uint64_t)xsm[xi][w + 1] : 0ull) << 32);
        const uint64_t hi = w + 2 < 4 ? (uint64_t)xsm[xi][w + 2] : 0ull;
        return sh == 0 ? lo : ((lo >> sh) | (hi << (64 - sh)));
      };
      for (int c = 0; c < nch; ++c) {
        int slot, cat, xi;
        key_info(c, slot, cat, xi);
        const uint64_t vm = vis_bits(cat, xi);
        const int pidx = 2 * c + (t >> 6);
        const bool loaded = pidx < npages && pgp[pidx] >= 0;
        const uint32_t idx = s0 + nch + c;
        const uint32_t sb = idx & 1;
        wait_bar(ctrl, &ctrl->s_full[sb], (idx >> 1) & 1, a.err, 21);
        ptx::tc_fence_after();
        const uint32_t sbase = tmem + tl + (sb ? TM_S1 : TM_S0) + (uint32_t)c0;
        float v[64];
        ptx::tmem_ld32(sbase, v);
        if (NC > 32) ptx::tmem_ld32(sbase + 32, v + 32);
        // The P^T buffer is free once the previous P.V product completed
        // (pv_done counts the two-pass chunks only; earlier resident chunks'
        // products completed before this sequence began, at that sequence's
        // o_done).
        const uint32_t pidx_g = opcount + c;
        if (pidx_g > 0) wait_bar(ctrl, &ctrl->pv_done, (pidx_g - 1) & 1, a.err, 23);
        ptx::tmem_ld_wait();
        // the scores are in registers: the TMEM buffer can take S^T of chunk c + 2
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&ctrl->s_empty[sb]);
        uint8_t* pth = smem + PT_OFF;
        uint8_t* ptl = pth + ptl_off;
        float mass2[2] = {0.f, 0.f};
#pragma unroll
        for (int g8 = 0; g8 < 8; ++g8) {
          if (8 * g8 < NC) {
            const float4* l4 = reinterpret_cast<const float4*>(ctrl->lse2 + c0 + 8 * g8);
            uint32_t ph[4], pq[4];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
              const float4 ll = l4[jj];
              const int j = 8 * g8 + 4 * jj;
              const float e0 = ptx::ex2(fmaf(v[j], sl2, -ll.x));
              const float e1 = ptx::ex2(fmaf(v[j + 1], sl2, -ll.y));
              const float e2 = ptx::ex2(fmaf(v[j + 2], sl2, -ll.z));
              const float e3 = ptx::ex2(fmaf(v[j + 3], sl2, -ll.w));
              const float q0 = ((vm >> j) & 1ull) ? e0 : 0.f;
              const float q1 = ((vm >> (j + 1)) & 1ull) ? e1 : 0.f;
              const float q2 = ((vm >> (j + 2)) & 1ull) ? e2 : 0.f;
              const float q3 = ((vm >> (j + 3)) & 1ull) ? e3 : 0.f;
              mass2[jj] += (q0 + q1) + (q2 + q3);
              ptx::split_bf16(q0, q1, ph[2 * jj], pq[2 * jj]);
              ptx::split_bf16(q2, q3, ph[2 * jj + 1], pq[2 * jj + 1]);
            }
            const int nb = (c0 >> 3) + g8;     // 8-row block of the sequence
            *reinterpret_cast<uint4*>(pth + nb * 2048 + t * 16) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
            *reinterpret_cast<uint4*>(ptl + nb * 2048 + t * 16) = make_uint4(pq[0], pq[1], pq[2], pq[3]);
          }
        }
        // both halves add into the zeroed mass row; two addends, so the
        // result does not depend on their order
        if (part && cat != 0) atomicAdd(part + slot, mass2[0] + mass2[1]);
        // V rows of keys nobody attends may hold anything (page tails):
        // zero them so that 0 * V stays 0 in the P.V product (each half
        // clears one 64-dimension half of the row).
        const uint32_t vitem = item_v2(c);
        const int vs = vitem % NSLOT;
        if (loaded && cat == 0) {
          wait_bar(ctrl, &ctrl->afull[vs], (vitem / NSLOT) & 1, a.err, 22);
          uint8_t* vrow = smem + SLOT_OFF + vs * SLOT_BYTES + half * HALF_BYTES +
                          (t >> 6) * BOX_BYTES + (t & 63) * 128;
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(vrow + ch * 16) = z;
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&ctrl->p_full);
      }
      }   // two-pass scheme
      // ----- O^T -> out (thread t = head dimension t; the halves split
      // rows): the sum of the hi and lo column ranges
      const int nsub_o = N16 >> 4;
      const uint32_t o_col = res ? 0u : TM_O;
      wait_bar(ctrl, &ctrl->o_done, ocount & 1, a.err, 24);
      ptx::tc_fence_after();
      if (!a.out_bf16) {
        float* o32 = static_cast<float*>(a.out);
        for (int k = half; k < nsub_o; k += 2) {
          float v[16];
          ptx::tmem_ld16(tmem + tl + o_col + 16 * k, v);
          float w2[16];
          ptx::tmem_ld16(tmem + tl + o_col + (uint32_t)N16 + 16 * k, w2);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] += w2[j];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int rr = 16 * k + j;
            if (rr < n) o32[(size_t)(gr0 + rr) * H + h * D + t] = any_page ? v[j] : 0.f;
          }
        }
      } else {
        __nv_bfloat16* o16 = static_cast<__nv_bfloat16*>(a.out);
        for (int k = half; k < nsub_o; k += 2) {
          float v[16];
          ptx::tmem_ld16(tmem + tl + o_col + 16 * k, v);
          float w2[16];
          ptx::tmem_ld16(tmem + tl + o_col + (uint32_t)N16 + 16 * k, w2);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] += w2[j];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int rr = 16 * k + j;
            if (rr < n)
              o16[(size_t)(gr0 + rr) * H + h * D + t] = __float2bfloat16_rn(any_page ? v[j] : 0.f);
          }
        }
      }
      ptx::tc_fence_before();
      // this sequence's TMEM is free for the next sequence's products
      __syncwarp();
      if (give_free && lane == 0) ptx::mbar_arrive(&ctrl->t_free);
    }
    ring = r0 + (res ? 2 : 3) * nch;
    scount = s0 + (res ? 0 : 2 * nch);
    ++ocount;
    if (!wide && !res) ++qcount;
    if (res) {
      ++rcount;
      rpcount += nch;
    } else {
      opcount += nch;
    }
    if (give_free) ++tcount;
  }

  // ================================================================ tile end
  // Before the next tile's projection reuses shared memory and TMEM, and
  // before TMEM is freed: every tcgen05 operation of this tile has completed
  // (the second completion of mma_done in the tile) and the last chunk loads
  // have landed (they have, unless a wait timed out).
  if (warp == kMmaWarp && lane == 0) {
    ptx::umma_commit(&ctrl->mma_done);
    ptx::mbar_wait(&ctrl->mma_done, 1, WAIT_NS);
  }
  if (warp == kProducerWarp && lane == 0 && ring > 0) {
    // only loads that were issued (none after a timeout)
    for (uint32_t it = ring > NSLOT ? ring - NSLOT : 0; it < ring; ++it)
      if ((int64_t)it <= last_load)
        ptx::mbar_wait(&ctrl->afull[it % NSLOT], (it / NSLOT) & 1, WAIT_NS);
  }
  __syncwarp();
  if constexpr (kPersist) {
    fence_async_smem();   // st.shared of this tile before the next tile's TMA writes
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    kstep0 += kb1 - kb0;
  }
  }   // tiles

  // ================================================================ teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, TMEM_COLS);
  // no rank leaves while another may still arrive on its shared memory
  if constexpr (kSplit) ptx::cluster_sync();
}

template <bool kPersist, bool kSplit, typename Sched>
cudaError_t launch_kernel(int grid, const StepPlan& plan, const Sched& sched, const StepArgs& a,
                          const void* const* tmap_x, const void* tmap_w, const void* tmap_k,
                          const void* tmap_v, cudaStream_t stream) {
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = opt_in_smem(reinterpret_cast<const void*>(step_bf16_kernel<kPersist, kSplit>),
                              SMEM_BYTES, attr_done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (kSplit) {   // one cluster of CL_RANKS CTAs per tile
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL_RANKS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, step_bf16_kernel<kPersist, kSplit>, plan, sched, a,
                            *reinterpret_cast<const CUtensorMap*>(tmap_x[0]),
                            *reinterpret_cast<const CUtensorMap*>(tmap_x[1]),
                            *reinterpret_cast<const CUtensorMap*>(tmap_x[2]),
                            *reinterpret_cast<const CUtensorMap*>(tmap_x[3]),
                            *reinterpret_cast<const CUtensorMap*>(tmap_w),
                            *reinterpret_cast<const CUtensorMap*>(tmap_k),
                            *reinterpret_cast<const CUtensorMap*>(tmap_v));
}

}  // namespace

size_t step_bf16_smem_bytes() { return SMEM_BYTES; }

bool step_bf16_split_ok(int tiles, int hidden, int sms) {
  return tiles > 0 && sms > 0 && CL_RANKS * tiles <= sms && hidden % (CL_RANKS * BK) == 0;
}

cudaError_t launch_step_bf16(const StepPlan& plan, const TileSched& sched, const StepArgs& a,
                             const void* const* tmap_x, const void* tmap_w, const void* tmap_k,
                             const void* tmap_v, bool split, cudaStream_t stream) {
  if (sched.n_bins > 0)
    return launch_kernel<true, false>(sched.n_bins, plan, sched, a, tmap_x, tmap_w, tmap_k,
                                      tmap_v, stream);
  const int grid = plan.n_groups * a.n_heads;
  if (grid == 0) return cudaSuccess;
  if (split)
    return launch_kernel<false, true>(CL_RANKS * grid, plan, NoSched{0}, a, tmap_x, tmap_w,
                                      tmap_k, tmap_v, stream);
  return launch_kernel<false, false>(grid, plan, NoSched{0}, a, tmap_x, tmap_w, tmap_k, tmap_v,
                                     stream);
}

}  // namespace fdllm
