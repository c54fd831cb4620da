/*
 * fdllm.h - C ABI of the Flash-dLLM per-layer hot path on NVIDIA B200 (sm_100a).
 *
 * One layer step of masked-diffusion decoding with Flash-dLLM KV caching:
 *   (a) Flash-Cache: the selected rows' hidden states go through the QKV
 *       projection, RoPE is applied, and K/V are written from on-chip memory
 *       straight into a paged KV cache; Q never leaves the SM.
 *   (b) scheduled attention: each sequence's query rows attend over that
 *       sequence's pages through its block table, so one launch covers a
 *       batch whose sequences differ in length and in stage; the Flash-Verify
 *       two-view mask is applied inside the same kernel, and each key's
 *       accumulated attention mass is emitted for the next step's top-k
 *       tracking set.
 *
 * Sources (cited by page title and paragraph):
 *   [FD] "Flash-dLLM: I/O-Aware KV Caching and Parallel Decoding for Fast,
 *        Memory-Efficient Diffusion LLMs" (ai4snews summary of the full text).
 *        Paragraph 1: Flash-Cache fuses QKV projection, RoPE and the cache
 *        write; scheduled Flash Attention aligns query blocks with their KV
 *        blocks through a block table across caching and update stages.
 *        Paragraph 2: each step's queries are a sliding unmasking window plus
 *        a fixed tracking budget of most-attended tokens.
 *        Paragraph 3: Flash-Verify places a draft view and a mask view at the
 *        same positions, sharing positional embeddings, isolated from each
 *        other by a causal mask inside the fused kernel.
 *   [AB] "Flash-dLLM: IO-Aware KV Caching and Parallel Decoding for Fast,
 *        Memory-Efficient Diffusion LLMs" (arXiv abstract page), Abstract:
 *        GPU memory I/O is the dominant bottleneck; an I/O-aware fused
 *        KV-cache kernel reduces redundant memory movement.
 *
 * Conventions for every entry point:
 *   - Pointers documented DEVICE are CUDA device pointers owned by the
 *     caller and borrowed for the duration of the call (and of the work it
 *     enqueues). Pointers documented HOST are read before the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Work is enqueued asynchronously; nothing synchronises except
 *     fdllm_check, fdllm_cache_create and steps run with validate = 1.
 *   - Host-detectable errors return a status and enqueue nothing.
 *     fdllm_last_error() returns a message for the calling thread.
 *   - Device-detected errors (a page id outside the pool, a slot past the
 *     block table, a position outside the RoPE table) skip the offending
 *     row, never trap, and are reported by the next fdllm_check as
 *     FDLLM_ERR_DEVICE_BOUNDS.
 *   - The library is single-GPU: every pointer must live on the device that
 *     was current at fdllm_cache_create.
 */
#ifndef FDLLM_H
#define FDLLM_H

#include <stdint.h>

#if defined(__GNUC__)
#define FDLLM_API __attribute__((visibility("default")))
#else
#define FDLLM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FDLLM_OK = 0,
  FDLLM_ERR_INVALID_ARG = 1,   /* bad pointer, size or shape (host check) */
  FDLLM_ERR_UNSUPPORTED = 2,   /* valid request outside what the kernels cover */
  FDLLM_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
  FDLLM_ERR_DEVICE_BOUNDS = 4, /* a kernel found out-of-range metadata */
  FDLLM_ERR_TIMEOUT = 5        /* a bounded in-kernel wait gave up */
} fdllm_status;

typedef enum { FDLLM_BF16 = 0, FDLLM_F32 = 1 } fdllm_dtype;

/* Shape of the paged KV cache and of the layer it serves.
 *   n_layers, n_heads, head_dim, page_size, num_pages: pool geometry.
 *   hidden = n_heads * head_dim (no grouped-query attention).
 *   max_position: RoPE positions must lie in [0, max_position).
 *   rope_theta: RoPE base (rotate-half pairing (i, i + head_dim/2), angle
 *     p * rope_theta^(-2i/head_dim); [FD] paragraph 1 fuses RoPE with the
 *     projection, the form is the LLaMA-family one).
 *   max_batch, max_slots_per_seq: bounds used to size the library's
 *     attention-mass workspace (n_heads * max_batch * max_slots_per_seq
 *     floats). A step with batch > max_batch or
 *     max_blocks_per_seq * page_size > max_slots_per_seq is rejected.
 *   dtype: FDLLM_BF16 (x, Wqkv, pools in bf16; fp32 accumulation) or
 *     FDLLM_F32 (everything fp32). */
typedef struct {
  int32_t n_layers;
  int32_t n_heads;
  int32_t head_dim;
  int32_t page_size;
  int32_t num_pages;
  int32_t max_position;
  int32_t max_batch;
  int32_t max_slots_per_seq;
  float rope_theta;
  int32_t dtype; /* fdllm_dtype */
} fdllm_cache_config;

typedef struct fdllm_cache fdllm_cache; /* opaque */

/* Per-step description.
 *   batch: sequences in the step (1 .. 256).
 *   total_rows: R = cu_rows[batch].
 *   max_blocks_per_seq: row length of block_table.
 *   cu_rows: HOST int32 [batch+1], row offsets of each sequence into x/out;
 *     a sequence holds at most 128 rows.
 *   seq_lens: HOST int32 [batch], L_b = visible context slots of sequence b
 *     (slots [0, L_b) through its block table).
 *   slots: DEVICE int32 [total_rows], cache slot each row writes; NULL means
 *     slot = position.
 *   validate: 1 = copy the device metadata to the host and check it before
 *     launching (slow; for tests). Duplicate slots within a sequence and
 *     view rows writing inside [0, L_b) are only detected this way.
 *   out_bf16: 0 = `out` is fp32; 1 = `out` is bf16, each value rounded to
 *     nearest even from the kernel's fp32 result (bf16 caches only; the
 *     input of fdllm_oproj). */
typedef struct {
  int32_t batch;
  int32_t total_rows;
  int32_t max_blocks_per_seq;
  const int32_t* cu_rows;
  const int32_t* seq_lens;
  const int32_t* slots;
  int32_t validate;
  int32_t out_bf16;
} fdllm_step;

/* Creates a handle over caller-owned pools.
 *   k_pool, v_pool: DEVICE [n_layers][num_pages][n_heads][page_size][head_dim]
 *     of cfg->dtype, 16-byte aligned. Not modified here.
 * Allocates the RoPE cos/sin tables (computed on the host in double and
 * kept in double: the kernels rotate q and k in double, so each rotated
 * value is rounded to the cache dtype once), the mass workspace and a
 * device error word, and synchronises `stream` once. */
FDLLM_API fdllm_status fdllm_cache_create(const fdllm_cache_config* cfg, void* k_pool, void* v_pool,
                                void* stream, fdllm_cache** out);

/* Frees what fdllm_cache_create allocated (not the pools). NULL is a no-op. */
FDLLM_API void fdllm_cache_destroy(fdllm_cache* cache);

/* One Flash-Cache + scheduled-attention layer step ([FD] paragraphs 1-3).
 *   layer: which layer's slice of the pools to write and read.
 *   x: DEVICE [total_rows][hidden] of the cache dtype, the selected rows'
 *     hidden states (window rows, tracked rows, or the two views).
 *   wqkv: DEVICE [hidden][3*hidden] row-major; columns are [Q | K | V], each
 *     block head-major (head h at columns h*head_dim .. +head_dim-1).
 *   positions: DEVICE int32 [total_rows], RoPE positions.
 *   block_table: DEVICE int32 [batch][max_blocks_per_seq], physical page of
 *     each logical page (slot s of sequence b lives in page
 *     block_table[b][s / page_size] at offset s % page_size).
 *   view_mask: DEVICE int8 [total_rows]: 0 plain row, 1 draft view, 2 mask
 *     view; NULL = all plain. Every row sees the slots [0, L_b) as they
 *     stand after this step's writes. A view row also sees the slots that
 *     rows of its own view write in this step at positions <= its own; the
 *     two views never see each other's fresh slots. View rows must write
 *     slots >= L_b.
 *   out: DEVICE [total_rows][hidden], fp32 (or bf16 with step->out_bf16),
 *     softmax(q k^T / sqrt(head_dim)) v per head, heads concatenated.
 *   attn_mass: DEVICE fp32 [batch][max_blocks_per_seq * page_size] or NULL.
 *     attn_mass[b][s] = (1 / (R_b * n_heads)) * sum over heads and over the
 *     rows of b of the attention probability on slot s; zero for slots
 *     nobody attends. Each sequence with rows sums to 1 ([FD] paragraph 2:
 *     the statistic behind the most-attended tracking set).
 * Writes: out, attn_mass, and for every row the k/v of every head into its
 * slot; no other cache byte changes. Within one step no sequence may read a
 * slot another sequence writes.
 * A handle's device workspace (mass partials, error word) serves one step
 * at a time: steps on one handle must not run concurrently (issue them on
 * one stream, or order the streams).
 * Steps with few tiles (four CTAs per tile fit on the SMs, e.g. a single
 * sequence; hidden a multiple of 256) run each tile as a cluster of four
 * CTAs that split the projection's K range and exchange partial sums
 * through distributed shared memory; the attending CTA waits, bounded to
 * one second, for the two CTAs that write the tile's k and v rows to the
 * cache. The four CTAs of a cluster are scheduled together, so the wait
 * only runs out if that work stalls: the tile's out and attn_mass are then
 * wrong and the step records FDLLM_ERR_TIMEOUT in the device error word.
 * With step->validate = 0 the call itself still returns FDLLM_OK, so
 * callers must call fdllm_check to see it. */
FDLLM_API fdllm_status fdllm_layer_step(fdllm_cache* cache, int32_t layer, const fdllm_step* step,
                              const void* x, const void* wqkv, const int32_t* positions,
                              const int32_t* block_table, const int8_t* view_mask, void* out,
                              float* attn_mass, void* stream);

/* Next step's tracked set ([FD] paragraph 2: a fixed budget of the most
 * attended tokens).
 *   attn_mass: DEVICE fp32 [batch][row_stride], non-negative.
 *   seq_lens: DEVICE int32 [batch]; candidates are slots [0, L_b), L_b <= row_stride,
 *     L_b <= 65536.
 *   k: budget, 1 .. 1024.
 *   exclude_cu: DEVICE int32 [batch+1] or NULL; exclude_slots: DEVICE int32,
 *     slots removed from sequence b's candidates are
 *     exclude_slots[exclude_cu[b] .. exclude_cu[b+1]) (out-of-range entries
 *     are ignored).
 *   tracked: DEVICE int32 [batch][k]: the k candidates of largest mass in
 *     descending order, ties to the lower slot, padded with -1. */
FDLLM_API fdllm_status fdllm_select_tracked(const float* attn_mass, const int32_t* seq_lens, int32_t batch,
                                  int32_t row_stride, int32_t k, const int32_t* exclude_cu,
                                  const int32_t* exclude_slots, int32_t* tracked, void* stream);

/* The layer step of fdllm_layer_step without a handle and without any
 * device allocation. The paper has no counterpart: it exists for callers
 * that cannot call cudaMalloc when they run a step, such as a serving
 * engine that has already given nearly all free HBM to its KV pool, or a
 * framework whose own allocator must account for every device byte.
 *   cfg, k_pool, v_pool: as for fdllm_cache_create (same rules).
 *   rope_cos, rope_sin: DEVICE fp64 [cfg->max_position][cfg->head_dim / 2],
 *     16-byte aligned, owned by the caller: entry [p][i] is the cosine / sine
 *     of p * rope_theta^(-2i/head_dim) in double (the tables that
 *     fdllm_cache_create builds).
 *   layer, step, x, wqkv, positions, block_table, view_mask, out, attn_mass,
 *     stream: as for fdllm_layer_step; cfg->max_batch and
 *     cfg->max_slots_per_seq bound the step the same way.
 * Scratch: the per-head attention-mass partials and the device error word
 * live in one fixed 8 MiB array in the library's device image, which every
 * GPU that loads the library holds until the process exits. With attn_mass
 * non-NULL, n_heads * batch * max_blocks_per_seq * page_size must be at most
 * 2,097,088 floats, else FDLLM_ERR_UNSUPPORTED (nothing enqueued).
 * The first call on each device looks up the array's device address and
 * clears its error word, synchronising `stream` once; make that first call
 * before any stream capture. Later calls enqueue work only (no host sync
 * unless step->validate is 1).
 * Every call on a device shares the array, so calls whose work overlaps on
 * the GPU (other streams, other threads) race on it and give wrong mass or
 * error reports; serialise them. The partial rows a call uses are zeroed by
 * its own kernel, so contents left by an earlier call do not matter.
 * Errors: device-detected errors are kept in the shared error word and
 * reported, then cleared, by the next call with step->validate = 1
 * (FDLLM_ERR_DEVICE_BOUNDS or FDLLM_ERR_TIMEOUT); fdllm_check does not see
 * them. No cudaMalloc, cudaFree or other device allocation happens; host
 * planning uses ordinary host memory as in fdllm_layer_step. */
FDLLM_API fdllm_status fdllm_layer_step_noalloc(const fdllm_cache_config* cfg, void* k_pool,
                                      void* v_pool, const double* rope_cos, const double* rope_sin,
                                      int32_t layer, const fdllm_step* step, const void* x,
                                      const void* wqkv, const int32_t* positions,
                                      const int32_t* block_table, const int8_t* view_mask,
                                      void* out, float* attn_mass, void* stream);

/* Flash-Verify acceptance ([FD] paragraph 3: a block position is accepted
 * only when the draft view and the mask view agree and the mask view's
 * confidence exceeds a threshold, in causal order, stopping at the first
 * position that fails).
 *   mask_logits: DEVICE [rows][vocab] of `dtype` (FDLLM_BF16 or FDLLM_F32):
 *     the mask view's logits at the block positions; the rows of sequence b
 *     are cu_rows[b] .. cu_rows[b+1]-1, in position order. Logits must be
 *     finite or -inf, with at least one finite value per row.
 *   cu_rows: DEVICE int32 [batch+1], non-decreasing, within [0, rows].
 *   draft_tokens: DEVICE int32 [rows], the drafted token at each position.
 *   tau: confidence threshold; acceptance needs conf > tau (compared in fp32).
 *   pred: DEVICE int32 [rows] out: the most likely token (lowest id among
 *     equal largest logits).
 *   conf: DEVICE fp32 [rows] out: that token's softmax probability.
 *   n_accepted: DEVICE int32 [batch] out: the length of the accepted prefix
 *     (positions i with pred == draft and conf > tau, from the first on).
 * Reads the logits once; two launches, asynchronous on `stream`. */
FDLLM_API fdllm_status fdllm_verify_accept(const void* mask_logits, int32_t dtype, int32_t rows,
                                 int32_t vocab, const int32_t* cu_rows, int32_t batch,
                                 const int32_t* draft_tokens, float tau, int32_t* pred,
                                 float* conf, int32_t* n_accepted, void* stream);

/* Host-only: the static tile schedule the bf16 layer step uses when its
 * (row group, head) tiles outnumber the SMs. The step then launches one
 * persistent CTA per SM (per bin), which runs its bin's tiles one after
 * another; fdllm_layer_step builds this schedule itself (with the device's
 * SM count and its own per-group cost model, and caches it while the costs
 * repeat). This entry point exposes the packing for inspection and tests.
 *
 * [FD] paragraph 1 (scheduled attention over divergent lengths and stages
 * in one launch): the packing balances that launch across SMs; the pages
 * prescribe no particular packing.
 *
 *   group_cost: HOST double [n_groups], the modelled time of one tile of
 *     group g (every head's tile of a group costs the same); finite, >= 0.
 *   n_groups, n_heads: tile t = g * n_heads + h for group g, head h.
 *     At most 256 each, and n_groups * n_heads <= 1024.
 *   n_bins: number of bins (persistent CTAs), 1 .. 160.
 *   bin_start: HOST int32 [n_bins + 1] out: bin i runs
 *     tiles[bin_start[i] .. bin_start[i+1]), costliest first; bin_start[0]
 *     is 0 and bin_start[n_bins] is n_groups * n_heads.
 *   tiles: HOST int32 [n_groups * n_heads] out: every tile exactly once.
 * Packing: first-fit-decreasing into n_bins bins of the smallest capacity
 * that fits (bisection), then moves and swaps out of the fullest bin while
 * they lower it. Deterministic. Returns FDLLM_ERR_INVALID_ARG or
 * FDLLM_ERR_UNSUPPORTED outside these limits; needs no GPU. */
FDLLM_API fdllm_status fdllm_plan_tile_schedule(const double* group_cost, int32_t n_groups,
                                      int32_t n_heads, int32_t n_bins, int32_t* bin_start,
                                      int32_t* tiles);

/* Output projection of the attention block: y = residual + attn_out W_o,
 * bf16 in and out, fp32 accumulation (one tcgen05 GEMM launch).
 * [FD] paragraph 1 covers a layer up to the attention output; the
 * projection after it is the plain linear map over the heads' outputs side
 * by side, read with the conventions of wqkv (y = x W, row-major, no bias).
 * With a residual it closes the layer's attention sub-block as a
 * transformer's residual stream does (x_next = x + attn_out W_o), which is
 * how a stack of layer steps chains one layer's output into the next
 * layer's x.
 *   attn_out: DEVICE bf16 [rows][hidden], e.g. fdllm_layer_step's out with
 *     step->out_bf16 = 1. Must not overlap y.
 *   w_o: DEVICE bf16 [hidden][hidden], row-major. Must not overlap y.
 *   residual: DEVICE bf16 [rows][hidden] or NULL (no residual). It may be y
 *     itself (an in-place update of the residual stream), but may not
 *     overlap y otherwise.
 *   y: DEVICE bf16 [rows][hidden] out; each value is the fp32 sum
 *     (accumulator + residual) rounded once to nearest even.
 *   rows >= 0 (0 enqueues nothing); hidden a positive multiple of 256.
 *   All pointers 16-byte aligned.
 *   status: DEVICE int32 or NULL; a bounded in-kernel wait that gives up
 *     writes FDLLM_ERR_TIMEOUT there (and y is then incomplete); nothing
 *     else writes it.
 * Host-detectable errors return FDLLM_ERR_INVALID_ARG or
 * FDLLM_ERR_UNSUPPORTED and enqueue nothing. */
FDLLM_API fdllm_status fdllm_oproj(const void* attn_out, const void* w_o, const void* residual,
                                   void* y, int32_t rows, int32_t hidden, int32_t* status,
                                   void* stream);

/* Synchronises `stream`, reads and clears the handle's device error word.
 * Returns FDLLM_OK, FDLLM_ERR_DEVICE_BOUNDS, FDLLM_ERR_TIMEOUT or
 * FDLLM_ERR_CUDA. */
FDLLM_API fdllm_status fdllm_check(fdllm_cache* cache, void* stream);

/* Failure injection for tests of the error path (the paper has no
 * counterpart). Faults are made on the host; nothing here traps, faults or
 * hangs the GPU.
 *   FDLLM_INJECT_SPLIT_FLAG_TIMEOUT: in the next fdllm_layer_step on `cache`
 *     that runs its tiles as four-CTA clusters, the k / v writing CTAs
 *     withhold their signal to the attending CTA, whose wait is bounded to
 *     `wait_ns` nanoseconds (1 .. 1e9) instead of one second. When it runs out
 *     the CTA records FDLLM_ERR_TIMEOUT in the device error word and skips
 *     its attention, issuing no further load or product; that step's out
 *     rows are left unwritten and its attention mass is zero. The next
 *     fdllm_check returns FDLLM_ERR_TIMEOUT and clears the word; the handle
 *     stays usable. The injection applies once, and stays pending while
 *     steps do not split their tiles.
 *   FDLLM_INJECT_NONE: cancels a pending injection.
 * Returns FDLLM_ERR_INVALID_ARG for a null handle, an unknown kind or a
 * wait outside the range. */
typedef enum { FDLLM_INJECT_NONE = 0, FDLLM_INJECT_SPLIT_FLAG_TIMEOUT = 1 } fdllm_inject_kind;
FDLLM_API fdllm_status fdllm_inject_fault(fdllm_cache* cache, int32_t kind, int64_t wait_ns);

/* Static description of a status code. */
FDLLM_API const char* fdllm_status_string(fdllm_status status);

/* Message for the last failing call on this thread ("" if none). */
FDLLM_API const char* fdllm_last_error(void);

/* Number of kernel launches the last successful fdllm_layer_step,
 * fdllm_layer_step_noalloc, fdllm_select_tracked, fdllm_verify_accept or
 * fdllm_oproj call on this thread enqueued. */
FDLLM_API int32_t fdllm_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* FDLLM_H */
