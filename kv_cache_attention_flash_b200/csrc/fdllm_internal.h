// Internal declarations shared by the host API and the kernels.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

namespace fdllm {

constexpr int kMaxBatch = 256;        // sequences per step
constexpr int kMaxGroups = 256;       // 128-row groups per step
constexpr int kGroupRows = 128;       // rows per group (the MMA's M)
constexpr int kMaxSeqRows = 128;      // rows per sequence
constexpr int kBf16PageSize = 64;     // page size of the bf16 kernel's page gathers
constexpr int kBf16MaxPages = 512;    // logical pages per sequence (bf16 kernel)
constexpr int kBf16GroupPages = 1024; // attended pages per row group (bf16 kernel)

// Device error word layout (int32[4]).
enum DevErr : int {
  kDevOk = 0,
  kDevBadPage = 1,      // block table entry outside [0, num_pages)
  kDevBadSlot = 2,      // slot < 0 or past max_blocks_per_seq * page_size
  kDevBadPosition = 3,  // position outside [0, max_position)
  kDevTimeout = 4,      // a bounded wait gave up
};

// Step plan: built on the host from cu_rows/seq_lens, passed by value.
struct StepPlan {
  int batch;
  int total_rows;
  int n_groups;
  int max_blocks;        // block table row length
  int row_stride;        // max_blocks * page_size (mass row length)
  int layer;
  int group_seq0[kMaxGroups + 1];  // group g: sequences seq_order[group_seq0[g] .. group_seq0[g+1])
  int seq_order[kMaxBatch];        // sequences with rows, group by group
  int cu_rows[kMaxBatch + 1];
  int seq_lens[kMaxBatch];
  int seq_qoff[kMaxBatch];         // first q row of the sequence in its group's 128-row tile
                                   // (a multiple of 16)
};

// Static tile schedule of the bf16 step: CTA i runs tiles
// tile[bin0[i] .. bin0[i+1]) in order, each encoded g << 8 | h. With
// n_bins == 0 the one-tile kernel runs instead, CTA i on tile i (group-major
// order). The schedule travels as a kernel parameter, so it is kept small
// (a larger parameter block costs launch time).
constexpr int kMaxSchedTiles = 1024;
constexpr int kMaxSchedBins = 160;
struct TileSched {
  int n_bins;
  uint16_t bin0[kMaxSchedBins + 1];
  uint16_t tile[kMaxSchedTiles];
};

// Per-call device pointers and pool geometry.
struct StepArgs {
  const void* x;
  const void* wqkv;
  const int32_t* positions;
  const int32_t* slots;          // may be null: slot = position
  const int32_t* block_table;
  const int8_t* view;            // may be null: all plain
  void* out;                     // fp32, or bf16 when out_bf16
  float* mass_part;              // [n_heads][batch][row_stride] or null
  void* k_pool;
  void* v_pool;
  const double* rope_cos;        // [max_position][head_dim/2]
  const double* rope_sin;
  int* err;                      // device error word
  int hidden;
  int n_heads;
  int head_dim;
  int page_size;
  int num_pages;
  int max_position;
  int out_bf16;
  // cluster split-K tiles (few tiles): the k / v owners arrive on rank 0's
  // kv_ready barrier only when split_wait_epoch == split_epoch (a test sets
  // them apart to withhold the arrivals), and rank 0 waits at most
  // flag_wait_ns nanoseconds for them
  uint32_t split_epoch;
  uint32_t split_wait_epoch;
  uint64_t flag_wait_ns;
};

// Launchers (return cudaGetLastError()).
// y = residual + o W_o (residual may be null or y itself) in tiles of 128
// rows x bn (256 or 128) columns: tmap_o over o
// [rows][hidden] with 128-row boxes, tmap_w the 3-D view of W_o {64 columns,
// hidden K rows, hidden / 64 column blocks} with boxes of bn / 64 blocks.
cudaError_t launch_oproj(const void* tmap_o, const void* tmap_w, int bn, const void* residual,
                         void* y, int rows, int hidden, int32_t* status, cudaStream_t stream);
size_t oproj_smem_bytes();
// tmap_x: x tensor maps with boxes of 16, 32, 64 and 128 rows. split: one
// cluster of 4 CTAs per tile (the K range of the projection split four
// ways); only where step_bf16_split_ok(tiles, hidden, SM count) holds and
// the schedule is empty.
cudaError_t launch_step_bf16(const StepPlan& plan, const TileSched& sched, const StepArgs& a,
                             const void* const* tmap_x, const void* tmap_w, const void* tmap_k,
                             const void* tmap_v, bool split, cudaStream_t stream);
bool step_bf16_split_ok(int tiles, int hidden, int sms);
cudaError_t launch_step_f32(const StepPlan& plan, const StepArgs& a, cudaStream_t stream);
cudaError_t launch_mass_reduce(const StepPlan& plan, const float* part, float* mass, int n_heads,
                               cudaStream_t stream);
cudaError_t launch_select_tracked(const float* mass, const int32_t* seq_lens, int batch,
                                  int row_stride, int k, const int32_t* exclude_cu,
                                  const int32_t* exclude_slots, int32_t* tracked,
                                  cudaStream_t stream);

cudaError_t launch_verify_accept(const void* logits, bool bf16, int rows, int vocab,
                                 const int32_t* cu_rows, int batch, const int32_t* draft,
                                 float tau, int32_t* pred, float* conf, int32_t* n_accepted,
                                 cudaStream_t stream);

size_t step_bf16_smem_bytes();

// Opts `fn` into `bytes` of dynamic shared memory on the current device.
// The attribute lives in each device's context, so the record of which
// devices are done is per device (a bit per device id below 64; others set
// it on every launch). Setting it twice is harmless, so concurrent first
// calls need no lock.
inline cudaError_t opt_in_smem(const void* fn, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t{1} << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}

}  // namespace fdllm
