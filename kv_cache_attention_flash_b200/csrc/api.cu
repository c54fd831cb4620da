// Host side of the C ABI declared in include/fdllm.h: argument checks, the
// row-group plan, TMA descriptors, kernel launches and error reporting.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <queue>
#include <mutex>
#include <set>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "fdllm.h"
#include "fdllm_internal.h"

using namespace fdllm;

namespace {

// NVTX range over one API call, so that a profiler's timeline shows each
// entry point around the kernels it launched (no cost without a profiler).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Bound of a split tile's wait for its k / v owners (the other in-kernel
// waits use the same one second).
constexpr uint64_t kFlagWaitNs = 1000000000ull;

thread_local std::string g_last_error;
thread_local int32_t g_last_launches = 0;

fdllm_status fail(fdllm_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

fdllm_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FDLLM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows][cols] matrix, box
// [box_rows][64 columns], 128-byte swizzle, zero fill out of bounds.
bool encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Wqkv [H][3H] bf16 viewed in 5 dimensions (column c within a 64-column
// half, K row k, half, q/k/v block, head): element (c, k, half, blk, head)
// is Wqkv[k][blk * H + head * head_dim + half * 64 + c]. One box
// {64, 64, 2, blocks, 1} is one head's q, k and v columns (blocks = 3), or
// one of them (blocks = 1), for 64 K rows, written to shared memory as
// 8 KB [64 rows][128 B] sub-boxes (128-byte swizzle).
bool encode_wqkv_5d(CUtensorMap* map, const void* base, uint64_t hidden, uint64_t n_heads,
                    uint64_t head_dim, uint32_t blocks) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[5] = {64, hidden, head_dim / 64, 3, n_heads};
  cuuint64_t strides[4] = {3 * hidden * 2, 128, hidden * 2, head_dim * 2};
  cuuint32_t box[5] = {64, 64, (cuuint32_t)(head_dim / 64), blocks, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A row-major bf16 [hidden][hidden] matrix viewed in 3 dimensions (column
// within a 64-column block, row, column block): element (c, k, j) is
// W[k][64 j + c]. One box {64, 64, blocks} is 64 rows of 64 * blocks
// columns, written to shared memory as `blocks` 8 KB [64 rows][128 B]
// sub-boxes (128-byte swizzle).
bool encode_w_3d(CUtensorMap* map, const void* base, uint64_t hidden, uint32_t blocks) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, hidden, hidden / 64};
  cuuint64_t strides[2] = {hidden * 2, 128};
  cuuint32_t box[3] = {64, 64, blocks};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
      cached[dev] = n;
  }
  return cached[dev];
}

// First fit of items (in the given order) into P bins of capacity C; the
// leftmost bin with room is found in a max-tree of remaining capacities.
bool first_fit(const std::vector<double>& cost, int P, double C, std::vector<int>& bin_of) {
  int size = 1;
  while (size < P) size <<= 1;
  thread_local std::vector<double> tree;
  tree.assign(2 * size, -1.0);
  for (int i = 0; i < P; ++i) tree[size + i] = C;
  for (int i = size - 1; i >= 1; --i) tree[i] = std::max(tree[2 * i], tree[2 * i + 1]);
  bin_of.assign(cost.size(), -1);
  for (size_t it = 0; it < cost.size(); ++it) {
    const double w = cost[it];
    if (tree[1] < w) return false;
    int node = 1;
    while (node < size) node = tree[2 * node] >= w ? 2 * node : 2 * node + 1;
    bin_of[it] = node - size;
    tree[node] -= w;
    for (node >>= 1; node >= 1; node >>= 1) tree[node] = std::max(tree[2 * node], tree[2 * node + 1]);
  }
  return true;
}

// Local improvement of an assignment of items (costs `sorted`) to P bins:
// while the fullest bin can hand a tile to another bin (or trade it for a
// cheaper one) and end up below its old load without the other bin reaching
// it, do the move that lowers the pair's larger load the most. Returns the
// final largest load.
double improve_packing(const std::vector<double>& sorted, int P, std::vector<int>& best) {
  const int n_items = (int)sorted.size();
  std::vector<double> load(P, 0.0);
  for (int i = 0; i < n_items; ++i) load[best[i]] += sorted[i];
  std::vector<std::vector<int>> members(P);
  for (int i = 0; i < n_items; ++i) members[best[i]].push_back(i);
  for (int iter = 0; iter < 4 * n_items; ++iter) {
    const int M = (int)(std::max_element(load.begin(), load.end()) - load.begin());
    double best_peak = load[M];
    int bi = -1, bj = -1, bb = -1;
    for (int ii = 0; ii < (int)members[M].size(); ++ii) {
      const double wi = sorted[members[M][ii]];
      for (int b = 0; b < P; ++b) {
        if (b == M) continue;
        // move
        const double pk = std::max(load[M] - wi, load[b] + wi);
        if (pk < best_peak - 1e-9) {
          best_peak = pk;
          bi = ii, bj = -1, bb = b;
        }
        // swap with a cheaper tile of bin b
        for (int jj = 0; jj < (int)members[b].size(); ++jj) {
          const double wj = sorted[members[b][jj]];
          if (wj >= wi) continue;
          const double pk2 = std::max(load[M] - wi + wj, load[b] + wi - wj);
          if (pk2 < best_peak - 1e-9) {
            best_peak = pk2;
            bi = ii, bj = jj, bb = b;
          }
        }
      }
    }
    if (bi < 0) break;
    const int item = members[M][bi];
    members[M].erase(members[M].begin() + bi);
    load[M] -= sorted[item];
    if (bj >= 0) {
      const int other = members[bb][bj];
      members[bb].erase(members[bb].begin() + bj);
      load[bb] -= sorted[other];
      members[M].push_back(other);
      load[M] += sorted[other];
      best[other] = M;
    }
    members[bb].push_back(item);
    load[bb] += sorted[item];
    best[item] = bb;
  }
  return *std::max_element(load.begin(), load.end());
}

// Longest-processing-time list schedule: each item (in decreasing cost) to
// the least-loaded bin, lowest index among equals.
std::vector<int> lpt_packing(const std::vector<double>& sorted, int P) {
  std::vector<int> bin_of(sorted.size());
  std::priority_queue<std::pair<double, int>, std::vector<std::pair<double, int>>,
                      std::greater<std::pair<double, int>>>
      heap;
  for (int b = 0; b < P; ++b) heap.push({0.0, b});
  for (size_t i = 0; i < sorted.size(); ++i) {
    auto top = heap.top();
    heap.pop();
    bin_of[i] = top.second;
    heap.push({top.first + sorted[i], top.second});
  }
  return bin_of;
}

// Packs the n_heads tiles of each group (tile (g, h) costs gcost[g]) into P
// bins: first-fit-decreasing under the smallest capacity that fits (found by
// bisection), then local moves and swaps out of the fullest bin. Each bin
// lists its tiles costliest first. False when first fit never succeeds.
bool pack_tiles(const std::vector<double>& gcost, int n_heads, int P, TileSched& sched) {
  const int ng = (int)gcost.size();
  const int n_items = ng * n_heads;
  std::vector<double> cost(n_items);
  double total = 0.0, cmax = 0.0;
  for (int g = 0; g < ng; ++g)
    for (int hh = 0; hh < n_heads; ++hh) {
      cost[g * n_heads + hh] = gcost[g];
      total += gcost[g];
      cmax = std::max(cmax, gcost[g]);
    }
  // items in decreasing cost (groups arrive in decreasing work; the modelled
  // cost may order them slightly differently)
  std::vector<int> order(n_items);
  for (int i = 0; i < n_items; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return cost[x] > cost[y]; });
  std::vector<double> sorted(n_items);
  for (int i = 0; i < n_items; ++i) sorted[i] = cost[order[i]];
  std::vector<int> bin_of, best;
  double lo = std::max(cmax, total / P), hi = lo;
  bool fits = first_fit(sorted, P, hi, best);
  for (int tries = 0; tries < 64 && !fits; ++tries) {
    hi *= 1.05;
    fits = first_fit(sorted, P, hi, best);
  }
  if (!fits) return false;
  for (int it = 0; it < 10; ++it) {
    const double mid = 0.5 * (lo + hi);
    if (first_fit(sorted, P, mid, bin_of)) {
      hi = mid;
      best = bin_of;
    } else {
      lo = mid;
    }
  }
  // Both first fit and LPT list scheduling, each locally improved; the
  // better of the two (first fit wins ties). Neither start dominates.
  {
    std::vector<int> alt = lpt_packing(sorted, P);
    const double m_ff = improve_packing(sorted, P, best);
    const double m_lpt = improve_packing(sorted, P, alt);
    if (m_lpt < m_ff) best = alt;
  }
  // each bin's tiles costliest first (items are in decreasing cost order)
  std::vector<int> count(P + 1, 0);
  for (int i = 0; i < n_items; ++i) ++count[best[i] + 1];
  for (int b = 0; b < P; ++b) count[b + 1] += count[b];
  for (int b = 0; b <= P; ++b) sched.bin0[b] = (uint16_t)count[b];
  std::vector<int> fill(count.begin(), count.end() - 1);
  for (int i = 0; i < n_items; ++i) {
    const int item = order[i];
    const int g = item / n_heads, hh = item % n_heads;
    sched.tile[fill[best[i]]++] = (uint16_t)((g << 8) | hh);
  }
  sched.n_bins = P;
  return true;
}

// Static schedule of the bf16 step's (group, head) tiles over the SMs, so
// that the tiles of a persistent CTA add up to about the same modelled time
// on every SM (list scheduling in launch order leaves the SMs that draw
// three long tiles well behind). Cached while the group costs repeat (every
// layer of a step shares them). n_bins = 0 asks for the one-tile kernel.
const TileSched& tile_schedule(const std::vector<double>& gcost, int n_heads) {
  thread_local TileSched sched;
  thread_local std::vector<double> last_cost;
  thread_local int last_heads = -1, last_sm = -1;
  const int ng = (int)gcost.size();
  const int n_items = ng * n_heads;
  const int P = std::min(std::min(sm_count(), kMaxSchedBins), n_items);
  // a CTA per tile already when the tiles fit on the SMs at once
  if (ng == 0 || n_heads > 256 || ng > 256 || n_items > kMaxSchedTiles || P <= 0 ||
      P > kMaxSchedBins || n_items <= P) {
    sched.n_bins = 0;
    last_heads = -1;
    return sched;
  }
  if (last_heads == n_heads && last_sm == P && last_cost == gcost) return sched;
  if (!pack_tiles(gcost, n_heads, P, sched)) {
    sched.n_bins = 0;
    last_heads = -1;
    return sched;
  }
  last_cost = gcost;
  last_heads = n_heads;
  last_sm = P;
  return sched;
}

}  // namespace

struct fdllm_cache {
  fdllm_cache_config cfg;
  CUtensorMap tmap_k;   // pools viewed as [rows = layer/page/head/slot][head_dim] (bf16)
  CUtensorMap tmap_v;
  void* k_pool;
  void* v_pool;
  int device;
  double* rope_cos;
  double* rope_sin;
  float* mass_part;
  size_t mass_part_floats;
  int* err;
  uint32_t split_epoch;    // counts cluster split-K launches (failure injection sets the
                           // kernel's wait epoch apart from it)
  int32_t inject_kind;     // pending failure injection (fdllm_inject_fault), 0 = none
  int64_t inject_wait_ns;
};

extern "C" {

const char* fdllm_status_string(fdllm_status s) {
  switch (s) {
    case FDLLM_OK: return "ok";
    case FDLLM_ERR_INVALID_ARG: return "invalid argument";
    case FDLLM_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case FDLLM_ERR_CUDA: return "CUDA error";
    case FDLLM_ERR_DEVICE_BOUNDS: return "device-side metadata out of bounds";
    case FDLLM_ERR_TIMEOUT: return "bounded in-kernel wait timed out";
  }
  return "unknown status";
}

const char* fdllm_last_error(void) { return g_last_error.c_str(); }

int32_t fdllm_last_launch_count(void) { return g_last_launches; }

fdllm_status fdllm_cache_create(const fdllm_cache_config* cfg, void* k_pool, void* v_pool,
                                void* stream, fdllm_cache** out) {
  NvtxRange nvtx_range("fdllm_cache_create");
  if (!cfg || !out) return fail(FDLLM_ERR_INVALID_ARG, "cache_create: null cfg or out");
  *out = nullptr;
  if (!k_pool || !v_pool) return fail(FDLLM_ERR_INVALID_ARG, "cache_create: null pool");
  if ((reinterpret_cast<uintptr_t>(k_pool) | reinterpret_cast<uintptr_t>(v_pool)) & 15)
    return fail(FDLLM_ERR_INVALID_ARG, "cache_create: pools must be 16-byte aligned");
  const fdllm_cache_config& c = *cfg;
  if (c.n_layers <= 0 || c.n_heads <= 0 || c.head_dim <= 0 || c.page_size <= 0 ||
      c.num_pages <= 0 || c.max_position <= 0 || c.max_batch <= 0 || c.max_slots_per_seq <= 0)
    return fail(FDLLM_ERR_INVALID_ARG, "cache_create: sizes must be positive");
  if (!(c.rope_theta > 1.0f) || !std::isfinite(c.rope_theta))
    return fail(FDLLM_ERR_INVALID_ARG, "cache_create: rope_theta must be finite and > 1");
  if (c.dtype != FDLLM_BF16 && c.dtype != FDLLM_F32)
    return fail(FDLLM_ERR_INVALID_ARG, "cache_create: unknown dtype %d", c.dtype);
  if (c.head_dim % 2)
    return fail(FDLLM_ERR_INVALID_ARG, "cache_create: head_dim must be even (RoPE pairs)");
  if (c.dtype == FDLLM_BF16 && c.head_dim != 128)
    return fail(FDLLM_ERR_UNSUPPORTED, "cache_create: bf16 kernels serve head_dim 128 only");
  if (c.dtype == FDLLM_F32 && (c.head_dim > 128 || c.head_dim % 32))
    return fail(FDLLM_ERR_UNSUPPORTED, "cache_create: fp32 kernel serves head_dim 32/64/96/128");
  if (c.max_batch > kMaxBatch)
    return fail(FDLLM_ERR_UNSUPPORTED, "cache_create: max_batch > %d", kMaxBatch);
  if (c.dtype == FDLLM_BF16 && c.page_size != kBf16PageSize)
    return fail(FDLLM_ERR_UNSUPPORTED, "cache_create: bf16 kernels gather %d-slot pages",
                kBf16PageSize);
  if ((long long)c.n_layers * c.num_pages * c.n_heads * c.page_size >= (1ll << 31))
    return fail(FDLLM_ERR_UNSUPPORTED, "cache_create: pool has 2^31 or more slot rows");

  fdllm_cache* h = new fdllm_cache();
  h->cfg = c;
  h->k_pool = k_pool;
  h->v_pool = v_pool;
  if (c.dtype == FDLLM_BF16) {
    const uint64_t rows = (uint64_t)c.n_layers * c.num_pages * c.n_heads * c.page_size;
    if (!encode_bf16_2d(&h->tmap_k, k_pool, rows, (uint64_t)c.head_dim, (uint32_t)c.page_size) ||
        !encode_bf16_2d(&h->tmap_v, v_pool, rows, (uint64_t)c.head_dim, (uint32_t)c.page_size)) {
      delete h;
      return fail(FDLLM_ERR_CUDA, "cache_create: cuTensorMapEncodeTiled failed for the pools");
    }
  }
  cudaGetDevice(&h->device);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  // RoPE tables in double: cos / sin of the angle p * theta^(-2i/D). The
  // kernels rotate in double too, so that each rotated q / k value is
  // rounded once, from a double close enough to the exact rotation that its
  // bf16 (or fp32) code is the exactly rounded one.
  const int half = c.head_dim / 2;
  const size_t nt = (size_t)c.max_position * half;
  std::vector<double> cs(nt), sn(nt);
  for (int p = 0; p < c.max_position; ++p)
    for (int i = 0; i < half; ++i) {
      const double inv = std::pow((double)c.rope_theta, -2.0 * i / c.head_dim);
      const double phi = (double)p * inv;
      cs[(size_t)p * half + i] = std::cos(phi);
      sn[(size_t)p * half + i] = std::sin(phi);
    }
  h->mass_part_floats = (size_t)c.n_heads * c.max_batch * c.max_slots_per_seq;
  cudaError_t e;
  if ((e = cudaMalloc(&h->rope_cos, nt * sizeof(double))) != cudaSuccess ||
      (e = cudaMalloc(&h->rope_sin, nt * sizeof(double))) != cudaSuccess ||
      (e = cudaMalloc(&h->mass_part, h->mass_part_floats * sizeof(float))) != cudaSuccess ||
      (e = cudaMalloc(&h->err, 4 * sizeof(int))) != cudaSuccess) {
    fdllm_cache_destroy(h);
    return cuda_fail(e, "cache_create: cudaMalloc");
  }
  if ((e = cudaMemcpyAsync(h->rope_cos, cs.data(), nt * sizeof(double), cudaMemcpyHostToDevice,
                           st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(h->rope_sin, sn.data(), nt * sizeof(double), cudaMemcpyHostToDevice,
                           st)) != cudaSuccess ||
      (e = cudaMemsetAsync(h->err, 0, 4 * sizeof(int), st)) != cudaSuccess ||
      (e = cudaStreamSynchronize(st)) != cudaSuccess) {
    fdllm_cache_destroy(h);
    return cuda_fail(e, "cache_create: upload");
  }
  *out = h;
  return FDLLM_OK;
}

void fdllm_cache_destroy(fdllm_cache* h) {
  if (!h) return;
  cudaFree(h->rope_cos);
  cudaFree(h->rope_sin);
  cudaFree(h->mass_part);
  cudaFree(h->err);
  delete h;
}

static fdllm_status validate_device_metadata(const fdllm_cache* h, int layer, const fdllm_step* st,
                                             const int32_t* positions, const int32_t* block_table,
                                             const int8_t* view, cudaStream_t stream) {
  const int R = st->total_rows, B = st->batch, mb = st->max_blocks_per_seq;
  const int ps = h->cfg.page_size;
  std::vector<int32_t> pos(R), slots(R), bt((size_t)B * mb);
  std::vector<int8_t> vw(R, 0);
  cudaError_t e;
  if ((e = cudaStreamSynchronize(stream)) != cudaSuccess) return cuda_fail(e, "validate: sync");
  if (R > 0) {
    if ((e = cudaMemcpy(pos.data(), positions, R * 4, cudaMemcpyDeviceToHost)) != cudaSuccess)
      return cuda_fail(e, "validate: positions");
    if (st->slots) {
      if ((e = cudaMemcpy(slots.data(), st->slots, R * 4, cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "validate: slots");
    } else {
      slots = pos;
    }
    if (view && (e = cudaMemcpy(vw.data(), view, R, cudaMemcpyDeviceToHost)) != cudaSuccess)
      return cuda_fail(e, "validate: view");
  }
  if ((e = cudaMemcpy(bt.data(), block_table, bt.size() * 4, cudaMemcpyDeviceToHost)) !=
      cudaSuccess)
    return cuda_fail(e, "validate: block_table");
  (void)layer;
  for (int b = 0; b < B; ++b) {
    std::set<int> seen;
    const int L = st->seq_lens[b];
    for (int r = st->cu_rows[b]; r < st->cu_rows[b + 1]; ++r) {
      if (pos[r] < 0 || pos[r] >= h->cfg.max_position)
        return fail(FDLLM_ERR_INVALID_ARG, "validate: row %d position %d outside [0, %d)", r,
                    pos[r], h->cfg.max_position);
      if (slots[r] < 0 || slots[r] >= mb * ps)
        return fail(FDLLM_ERR_INVALID_ARG, "validate: row %d slot %d outside [0, %d)", r, slots[r],
                    mb * ps);
      if (vw[r] < 0 || vw[r] > 2)
        return fail(FDLLM_ERR_INVALID_ARG, "validate: row %d view %d not in {0,1,2}", r, vw[r]);
      if (vw[r] != 0 && slots[r] < L)
        return fail(FDLLM_ERR_INVALID_ARG, "validate: view row %d writes slot %d inside [0, %d)",
                    r, slots[r], L);
      if (!seen.insert(slots[r]).second)
        return fail(FDLLM_ERR_INVALID_ARG, "validate: sequence %d writes slot %d twice", b,
                    slots[r]);
      const int pg = bt[(size_t)b * mb + slots[r] / ps];
      if (pg < 0 || pg >= h->cfg.num_pages)
        return fail(FDLLM_ERR_INVALID_ARG, "validate: row %d slot %d maps to page %d", r,
                    slots[r], pg);
    }
    if (st->cu_rows[b + 1] > st->cu_rows[b])
      for (int i = 0; i < (L + ps - 1) / ps; ++i) {
        const int pg = bt[(size_t)b * mb + i];
        if (pg < 0 || pg >= h->cfg.num_pages)
          return fail(FDLLM_ERR_INVALID_ARG, "validate: sequence %d logical page %d -> %d", b, i,
                      pg);
      }
  }
  return FDLLM_OK;
}

fdllm_status fdllm_layer_step(fdllm_cache* h, int32_t layer, const fdllm_step* st, const void* x,
                              const void* wqkv, const int32_t* positions,
                              const int32_t* block_table, const int8_t* view_mask, void* out,
                              float* attn_mass, void* stream) {
  NvtxRange nvtx_range("fdllm_layer_step");
  if (!h || !st) return fail(FDLLM_ERR_INVALID_ARG, "layer_step: null handle or step");
  const fdllm_cache_config& c = h->cfg;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (layer < 0 || layer >= c.n_layers)
    return fail(FDLLM_ERR_INVALID_ARG, "layer_step: layer %d outside [0, %d)", layer, c.n_layers);
  if (st->batch <= 0 || st->batch > kMaxBatch)
    return fail(FDLLM_ERR_INVALID_ARG, "layer_step: batch %d outside [1, %d]", st->batch,
                kMaxBatch);
  if (st->batch > c.max_batch)
    return fail(FDLLM_ERR_INVALID_ARG, "layer_step: batch %d > max_batch %d", st->batch,
                c.max_batch);
  if (!st->cu_rows || !st->seq_lens)
    return fail(FDLLM_ERR_INVALID_ARG, "layer_step: cu_rows and seq_lens (host) are required");
  if (st->max_blocks_per_seq <= 0)
    return fail(FDLLM_ERR_INVALID_ARG, "layer_step: max_blocks_per_seq must be positive");
  const long long row_stride = (long long)st->max_blocks_per_seq * c.page_size;
  if (row_stride > c.max_slots_per_seq)
    return fail(FDLLM_ERR_INVALID_ARG,
                "layer_step: max_blocks_per_seq * page_size = %lld > max_slots_per_seq %d",
                row_stride, c.max_slots_per_seq);
  if (st->cu_rows[0] != 0 || st->cu_rows[st->batch] != st->total_rows)
    return fail(FDLLM_ERR_INVALID_ARG, "layer_step: cu_rows must run from 0 to total_rows");
  for (int b = 0; b < st->batch; ++b) {
    const int n = st->cu_rows[b + 1] - st->cu_rows[b];
    if (n < 0) return fail(FDLLM_ERR_INVALID_ARG, "layer_step: cu_rows decreases at %d", b);
    if (n > kMaxSeqRows)
      return fail(FDLLM_ERR_UNSUPPORTED, "layer_step: sequence %d has %d rows (> %d)", b, n,
                  kMaxSeqRows);
    if (st->seq_lens[b] < 0 || st->seq_lens[b] > row_stride)
      return fail(FDLLM_ERR_INVALID_ARG, "layer_step: seq_lens[%d] = %d outside [0, %lld]", b,
                  st->seq_lens[b], row_stride);
  }
  const int R = st->total_rows;
  if (R > 0 && (!x || !wqkv || !positions || !out))
    return fail(FDLLM_ERR_INVALID_ARG, "layer_step: null x, wqkv, positions or out");
  if (!block_table) return fail(FDLLM_ERR_INVALID_ARG, "layer_step: null block_table");
  const int H = c.n_heads * c.head_dim;
  if (c.dtype == FDLLM_BF16) {
    if (H % 64)
      return fail(FDLLM_ERR_UNSUPPORTED, "layer_step: hidden %d not a multiple of 64", H);
    if (st->max_blocks_per_seq > kBf16MaxPages)
      return fail(FDLLM_ERR_UNSUPPORTED, "layer_step: more than %d pages per sequence",
                  kBf16MaxPages);
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(wqkv)) & 15)
      return fail(FDLLM_ERR_INVALID_ARG, "layer_step: x and wqkv must be 16-byte aligned");
  }
  if (reinterpret_cast<uintptr_t>(out) & 15)
    return fail(FDLLM_ERR_INVALID_ARG, "layer_step: out must be 16-byte aligned");
  if (st->out_bf16 != 0 && st->out_bf16 != 1)
    return fail(FDLLM_ERR_INVALID_ARG, "layer_step: out_bf16 must be 0 or 1");
  if (st->out_bf16 && c.dtype != FDLLM_BF16)
    return fail(FDLLM_ERR_UNSUPPORTED, "layer_step: bf16 out needs a bf16 cache");

  if (st->validate) {
    fdllm_status vs = validate_device_metadata(h, layer, st, positions, block_table, view_mask, s);
    if (vs != FDLLM_OK) return vs;
  }

  StepPlan plan;
  memset(&plan, 0, sizeof(plan));
  plan.batch = st->batch;
  plan.total_rows = R;
  plan.max_blocks = st->max_blocks_per_seq;
  plan.row_stride = (int)row_stride;
  plan.layer = layer;
  for (int b = 0; b <= st->batch; ++b) plan.cu_rows[b] = st->cu_rows[b];
  for (int b = 0; b < st->batch; ++b) plan.seq_lens[b] = st->seq_lens[b];
  std::vector<double> gcost;   // modelled tile duration of each group
  // Row groups (one 128-row tile each): whole sequences, each padded to a
  // multiple of 16 q rows (the attention MMA's N granularity), packed first
  // fit in order of decreasing size. The bf16 kernel also keeps a group's
  // attended page list on chip (at most kBf16GroupPages entries, bounded by
  // context pages + rows) and serves at most 8 sequences per group. Groups
  // are launched in order of decreasing attention work, head by head within
  // a group, so that the longest tiles start first and the short ones fill
  // in at the end. Work is counted in 128-key chunks (a chunk costs about
  // the same whatever the row count) plus one chunk per sequence.
  {
    struct Grp {
      int pad, pages;
      long long cost;
      std::vector<int> seqs;
    };
    gcost.clear();
    std::vector<int> idx;
    for (int b = 0; b < st->batch; ++b) {
      plan.seq_qoff[b] = 0;
      if (st->cu_rows[b + 1] > st->cu_rows[b]) idx.push_back(b);
    }
    auto rows_of = [&](int b) { return st->cu_rows[b + 1] - st->cu_rows[b]; };
    auto n16 = [&](int b) { return (rows_of(b) + 15) & ~15; };
    auto pages = [&](int b) {
      return (st->seq_lens[b] + c.page_size - 1) / c.page_size + rows_of(b);
    };
    auto work = [&](int b) -> long long {
      const int ctx = (st->seq_lens[b] + c.page_size - 1) / c.page_size;
      const int extra = (rows_of(b) + c.page_size - 1) / c.page_size + 1;
      return (ctx + extra + 1) / 2 + 1;
    };
    std::stable_sort(idx.begin(), idx.end(), [&](int x, int y) {
      if (n16(x) != n16(y)) return n16(x) > n16(y);
      return work(x) > work(y);
    });
    std::vector<Grp> groups;
    for (int b : idx) {
      Grp* dst = nullptr;
      for (auto& gp : groups)
        if (gp.pad + n16(b) <= kGroupRows && gp.pages + pages(b) <= kBf16GroupPages &&
            (int)gp.seqs.size() < kGroupRows / 16) {
          dst = &gp;
          break;
        }
      if (!dst) {
        groups.push_back(Grp{0, 0, 0, {}});
        dst = &groups.back();
      }
      dst->pad += n16(b);
      dst->pages += pages(b);
      dst->cost += work(b);
      dst->seqs.push_back(b);
    }
    if ((int)groups.size() > kMaxGroups)
      return fail(FDLLM_ERR_UNSUPPORTED, "layer_step: more than %d row groups", kMaxGroups);
    std::stable_sort(groups.begin(), groups.end(),
                     [](const Grp& x, const Grp& y) { return x.cost > y.cost; });
    int k = 0;
    for (size_t gi = 0; gi < groups.size(); ++gi) {
      plan.group_seq0[gi] = k;
      int off = 0;
      for (int b : groups[gi].seqs) {
        plan.seq_order[k++] = b;
        plan.seq_qoff[b] = off;
        off += n16(b);
      }
    }
    plan.group_seq0[groups.size()] = k;
    plan.n_groups = (int)groups.size();
    // Modelled duration of a group's tile on B200 (us, least-squares fits
    // to measured per-tile timelines): the projection grows with the number
    // of x boxes (one per power-of-two piece of each sequence's padded
    // rows), attention with the 128-key chunks, a little more for wider
    // sequences. Sequences whose scores stay resident in TMEM (16, 32 or 64
    // padded rows whose context chunks fit 512 columns) pay more per
    // sequence and less per chunk than the two-pass ones.
    for (const Grp& gp : groups) {
      int nbox = 0;
      double attn = 0.0;
      for (int b : gp.seqs) {
        nbox += __builtin_popcount((unsigned)(n16(b) / 16));
        const int ctx = (st->seq_lens[b] + c.page_size - 1) / c.page_size;
        const int extra = (rows_of(b) + c.page_size - 1) / c.page_size + 1;
        const int chunks = (ctx + extra + 1) / 2;
        const int w = n16(b);
        const bool resident = (w == 16 || w == 32 || w == 64) && ((ctx + 1) / 2) * w <= 512;
        attn += resident ? 1.58 + chunks * (1.61 + 0.319 * (w / 16))
                         : 0.53 + chunks * (2.58 + 0.144 * (w / 16));
      }
      gcost.push_back(59.2 + 2.0 * nbox + attn);
    }
  }
  const int ng = plan.n_groups;

  StepArgs a;
  a.x = x;
  a.wqkv = wqkv;
  a.positions = positions;
  a.slots = st->slots;
  a.block_table = block_table;
  a.view = view_mask;
  a.out = out;
  a.mass_part = attn_mass ? h->mass_part : nullptr;
  a.k_pool = h->k_pool;
  a.v_pool = h->v_pool;
  a.rope_cos = h->rope_cos;
  a.rope_sin = h->rope_sin;
  a.err = h->err;
  a.hidden = H;
  a.n_heads = c.n_heads;
  a.head_dim = c.head_dim;
  a.page_size = c.page_size;
  a.num_pages = c.num_pages;
  a.max_position = c.max_position;
  a.out_bf16 = st->out_bf16;
  a.split_epoch = 0;
  a.split_wait_epoch = 0;
  a.flag_wait_ns = kFlagWaitNs;

  int launches = 0;
  cudaError_t e = cudaSuccess;
  if (ng > 0) {
    if (c.dtype == FDLLM_BF16) {
      CUtensorMap tx[4], tw;
      const void* txp[4];
      for (int i = 0; i < 4; ++i) {
        if (!encode_bf16_2d(&tx[i], x, (uint64_t)R, (uint64_t)H, 16u << i))
          return fail(FDLLM_ERR_CUDA, "layer_step: cuTensorMapEncodeTiled failed (x)");
        txp[i] = &tx[i];
      }
      if (!encode_wqkv_5d(&tw, wqkv, (uint64_t)H, (uint64_t)c.n_heads, (uint64_t)c.head_dim, 3))
        return fail(FDLLM_ERR_CUDA, "layer_step: cuTensorMapEncodeTiled failed (wqkv)");
      const TileSched& ts = tile_schedule(gcost, c.n_heads);
      // Few tiles: a cluster of four CTAs per tile splits the projection's
      // K range, so that four times as many SMs stream the weights and
      // issue the products.
      const int tiles = ng * c.n_heads;
      const bool split = ts.n_bins == 0 && step_bf16_split_ok(tiles, H, sm_count());
      if (split) {
        ++h->split_epoch;
        a.split_epoch = h->split_epoch;
        a.split_wait_epoch = h->split_epoch;
        if (h->inject_kind == FDLLM_INJECT_SPLIT_FLAG_TIMEOUT) {
          // the k / v owners withhold their arrivals: rank 0's wait runs out
          a.split_wait_epoch = h->split_epoch ^ 0x80000000u;
          a.flag_wait_ns = (uint64_t)h->inject_wait_ns;
          h->inject_kind = 0;
        }
      }
      e = launch_step_bf16(plan, ts, a, txp, &tw, &h->tmap_k, &h->tmap_v, split, s);
    } else {
      e = launch_step_f32(plan, a, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "layer_step: step kernel launch");
    ++launches;
  }
  if (attn_mass) {
    e = launch_mass_reduce(plan, h->mass_part, attn_mass, c.n_heads, s);
    if (e != cudaSuccess) return cuda_fail(e, "layer_step: mass reduce launch");
    ++launches;
  }
  g_last_launches = launches;
  if (st->validate) {
    if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e, "layer_step: sync");
  }
  return FDLLM_OK;
}

fdllm_status fdllm_select_tracked(const float* attn_mass, const int32_t* seq_lens, int32_t batch,
                                  int32_t row_stride, int32_t k, const int32_t* exclude_cu,
                                  const int32_t* exclude_slots, int32_t* tracked, void* stream) {
  NvtxRange nvtx_range("fdllm_select_tracked");
  if (!attn_mass || !seq_lens || !tracked)
    return fail(FDLLM_ERR_INVALID_ARG, "select_tracked: null attn_mass, seq_lens or tracked");
  if (batch <= 0) return fail(FDLLM_ERR_INVALID_ARG, "select_tracked: batch must be positive");
  if (row_stride <= 0 || row_stride > 65536)
    return fail(FDLLM_ERR_UNSUPPORTED, "select_tracked: row_stride %d outside [1, 65536]",
                row_stride);
  if (k <= 0 || k > 1024)
    return fail(FDLLM_ERR_UNSUPPORTED, "select_tracked: k %d outside [1, 1024]", k);
  if ((exclude_cu == nullptr) != (exclude_slots == nullptr))
    return fail(FDLLM_ERR_INVALID_ARG, "select_tracked: exclude_cu and exclude_slots go together");
  cudaError_t e = launch_select_tracked(attn_mass, seq_lens, batch, row_stride, k, exclude_cu,
                                        exclude_slots, tracked,
                                        reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "select_tracked: launch");
  g_last_launches = 1;
  return FDLLM_OK;
}

fdllm_status fdllm_verify_accept(const void* mask_logits, int32_t dtype, int32_t rows,
                                 int32_t vocab, const int32_t* cu_rows, int32_t batch,
                                 const int32_t* draft_tokens, float tau, int32_t* pred,
                                 float* conf, int32_t* n_accepted, void* stream) {
  NvtxRange nvtx_range("fdllm_verify_accept");
  if (dtype != FDLLM_BF16 && dtype != FDLLM_F32)
    return fail(FDLLM_ERR_INVALID_ARG, "verify_accept: unknown dtype %d", dtype);
  if (rows < 0 || batch <= 0 || vocab <= 0)
    return fail(FDLLM_ERR_INVALID_ARG, "verify_accept: rows >= 0, batch > 0, vocab > 0 required");
  if (!cu_rows || !n_accepted)
    return fail(FDLLM_ERR_INVALID_ARG, "verify_accept: null cu_rows or n_accepted");
  if (rows > 0 && (!mask_logits || !draft_tokens || !pred || !conf))
    return fail(FDLLM_ERR_INVALID_ARG, "verify_accept: null logits, draft tokens, pred or conf");
  cudaError_t e = launch_verify_accept(mask_logits, dtype == FDLLM_BF16, rows, vocab, cu_rows,
                                       batch, draft_tokens, tau, pred, conf, n_accepted,
                                       reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "verify_accept: launch");
  g_last_launches = rows > 0 ? 2 : 1;
  return FDLLM_OK;
}

fdllm_status fdllm_plan_tile_schedule(const double* group_cost, int32_t n_groups,
                                      int32_t n_heads, int32_t n_bins, int32_t* bin_start,
                                      int32_t* tiles) {
  if (!group_cost || !bin_start || !tiles)
    return fail(FDLLM_ERR_INVALID_ARG, "plan_tile_schedule: null pointer");
  if (n_groups <= 0 || n_heads <= 0 || n_bins <= 0)
    return fail(FDLLM_ERR_INVALID_ARG, "plan_tile_schedule: sizes must be positive");
  if (n_groups > 256 || n_heads > 256 || n_groups * n_heads > kMaxSchedTiles ||
      n_bins > kMaxSchedBins)
    return fail(FDLLM_ERR_UNSUPPORTED,
                "plan_tile_schedule: at most 256 groups, 256 heads, %d tiles and %d bins",
                kMaxSchedTiles, kMaxSchedBins);
  std::vector<double> gc(group_cost, group_cost + n_groups);
  for (double v : gc)
    if (!(v >= 0.0) || !std::isfinite(v))
      return fail(FDLLM_ERR_INVALID_ARG, "plan_tile_schedule: costs must be finite and >= 0");
  TileSched ts;
  if (!pack_tiles(gc, n_heads, n_bins, ts))
    return fail(FDLLM_ERR_UNSUPPORTED, "plan_tile_schedule: no packing found");
  for (int b = 0; b <= n_bins; ++b) bin_start[b] = ts.bin0[b];
  for (int i = 0; i < n_groups * n_heads; ++i)
    tiles[i] = (ts.tile[i] >> 8) * n_heads + (ts.tile[i] & 255);
  return FDLLM_OK;
}

fdllm_status fdllm_oproj(const void* attn_out, const void* w_o, const void* residual, void* y,
                         int32_t rows, int32_t hidden, int32_t* status, void* stream) {
  NvtxRange nvtx_range("fdllm_oproj");
  if (rows < 0 || hidden <= 0)
    return fail(FDLLM_ERR_INVALID_ARG, "oproj: rows >= 0 and hidden > 0 required");
  if (hidden % 256)
    return fail(FDLLM_ERR_UNSUPPORTED, "oproj: hidden %d not a multiple of 256", hidden);
  if (rows == 0) {
    g_last_launches = 0;
    return FDLLM_OK;
  }
  if (!attn_out || !w_o || !y) return fail(FDLLM_ERR_INVALID_ARG, "oproj: null pointer");
  if ((reinterpret_cast<uintptr_t>(attn_out) | reinterpret_cast<uintptr_t>(w_o) |
       reinterpret_cast<uintptr_t>(residual) | reinterpret_cast<uintptr_t>(y)) & 15)
    return fail(FDLLM_ERR_INVALID_ARG, "oproj: pointers must be 16-byte aligned");
  {
    // y may be the residual itself, but overlaps no input otherwise
    const uintptr_t yb = reinterpret_cast<uintptr_t>(y);
    const uintptr_t ye = yb + (uintptr_t)rows * hidden * 2;
    auto overlaps = [&](const void* p, size_t bytes) {
      const uintptr_t b = reinterpret_cast<uintptr_t>(p);
      return b < ye && yb < b + bytes;
    };
    const size_t act = (size_t)rows * hidden * 2;
    if (overlaps(attn_out, act) || overlaps(w_o, (size_t)hidden * hidden * 2) ||
        (residual && residual != y && overlaps(residual, act)))
      return fail(FDLLM_ERR_INVALID_ARG, "oproj: y overlaps an input");
  }
  // Tile width: 256 columns unless 128-column tiles finish sooner. A
  // 128-wide tile does half the work but takes 0.87 of a 256-wide one's time
  // on B200 (26.6 vs 30.7 us at 1536 x 4096: the narrower MMA re-reads its A
  // operand from shared memory per half as many columns), so it only pays
  // when the 256-wide tiles would leave most SMs idle in their last wave.
  const int sms = sm_count() > 0 ? sm_count() : 148;
  const long long rt = (rows + 127) / 128;
  const long long w256 = (rt * (hidden / 256) + sms - 1) / sms;
  const long long w128 = (rt * (hidden / 128) + sms - 1) / sms;
  const int bn = (double)w128 * 0.87 < (double)w256 ? 128 : 256;
  CUtensorMap to, tw;
  if (!encode_bf16_2d(&to, attn_out, (uint64_t)rows, (uint64_t)hidden, 128u) ||
      !encode_w_3d(&tw, w_o, (uint64_t)hidden, (uint32_t)(bn / 64)))
    return fail(FDLLM_ERR_CUDA, "oproj: cuTensorMapEncodeTiled failed");
  cudaError_t e = launch_oproj(&to, &tw, bn, residual, y, rows, hidden, status,
                               reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "oproj: launch");
  g_last_launches = 1;
  return FDLLM_OK;
}

fdllm_status fdllm_inject_fault(fdllm_cache* h, int32_t kind, int64_t wait_ns) {
  if (!h) return fail(FDLLM_ERR_INVALID_ARG, "inject_fault: null handle");
  if (kind == FDLLM_INJECT_NONE) {
    h->inject_kind = 0;
    return FDLLM_OK;
  }
  if (kind != FDLLM_INJECT_SPLIT_FLAG_TIMEOUT)
    return fail(FDLLM_ERR_INVALID_ARG, "inject_fault: unknown kind %d", kind);
  if (wait_ns < 1 || wait_ns > (int64_t)kFlagWaitNs)
    return fail(FDLLM_ERR_INVALID_ARG, "inject_fault: wait_ns %lld outside [1, 1e9]",
                (long long)wait_ns);
  h->inject_kind = kind;
  h->inject_wait_ns = wait_ns;
  return FDLLM_OK;
}

fdllm_status fdllm_check(fdllm_cache* h, void* stream) {
  NvtxRange nvtx_range("fdllm_check");
  if (!h) return fail(FDLLM_ERR_INVALID_ARG, "check: null handle");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "check: sync");
  int w[4];
  if ((e = cudaMemcpy(w, h->err, sizeof(w), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "check: read error word");
  if (w[0] == 0) return FDLLM_OK;
  if ((e = cudaMemset(h->err, 0, sizeof(w))) != cudaSuccess)
    return cuda_fail(e, "check: clear error word");
  static const char* what[] = {"ok", "page id outside the pool", "slot past the block table",
                               "position outside the RoPE table", "bounded wait timed out"};
  const int code = (w[0] >= 0 && w[0] <= 4) ? w[0] : 0;
  if (code == kDevTimeout)
    return fail(FDLLM_ERR_TIMEOUT, "device: %s (site %d)", what[code], w[1]);
  return fail(FDLLM_ERR_DEVICE_BOUNDS, "device: %s (detail %d)", what[code], w[1]);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Layer step that allocates no device memory.
//
// Some callers cannot call cudaMalloc at the time they run a step: a serving
// engine that has already handed nearly all free HBM to its paged KV pool
// (a late cudaMalloc would fail or fragment that reservation), or a host
// framework whose own allocator must account for every device byte. For
// them the step's only scratch, the per-head attention-mass partial sums
// and the device error word, lives in the fixed array below, part of the
// library's device image, instead of in a handle's cudaMalloc'd workspace.
// The caller passes the pools and the RoPE tables it owns; nothing else is
// needed, so no handle is created.
//
// Layout of the array: bytes [0, 16) the error word (int32[4]; must start at
// zero: cleared on the first call on each device and after every report),
// bytes [256, end) the mass partials [n_heads][batch][max_blocks*page_size]
// fp32 (each row the step uses is zeroed by the kernel before it
// accumulates, so stale contents from an earlier call do not matter).

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB per device
constexpr size_t kNoAllocPartOffset = 256;
constexpr size_t kNoAllocPartFloats = (kNoAllocScratchBytes - kNoAllocPartOffset) / sizeof(float);
constexpr int kNoAllocMaxDevices = 64;

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoAllocMaxDevices];   // device address of the array, per device

// Device address of g_noalloc_scratch on the current device. The first call
// on a device looks it up (cudaGetSymbolAddress, with that device current),
// zeroes the error word on `stream` and waits for that; later calls reuse
// the address.
fdllm_status noalloc_scratch(cudaStream_t stream, void** addr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "layer_step_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return fail(FDLLM_ERR_UNSUPPORTED, "layer_step_noalloc: device ordinal %d >= %d", dev,
                kNoAllocMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_noalloc_scratch)) != cudaSuccess)
      return cuda_fail(e, "layer_step_noalloc: cudaGetSymbolAddress");
    if ((e = cudaMemsetAsync(p, 0, 4 * sizeof(int), stream)) != cudaSuccess ||
        (e = cudaStreamSynchronize(stream)) != cudaSuccess)
      return cuda_fail(e, "layer_step_noalloc: clear error word");
    g_noalloc_addr[dev] = p;
  }
  *addr = g_noalloc_addr[dev];
  return FDLLM_OK;
}

}  // namespace

extern "C" {

fdllm_status fdllm_layer_step_noalloc(const fdllm_cache_config* cfg, void* k_pool, void* v_pool,
                                      const double* rope_cos, const double* rope_sin, int32_t layer,
                                      const fdllm_step* st, const void* x, const void* wqkv,
                                      const int32_t* positions, const int32_t* block_table,
                                      const int8_t* view_mask, void* out, float* attn_mass,
                                      void* stream) {
  NvtxRange nvtx_range("fdllm_layer_step_noalloc");
  if (!cfg || !st) return fail(FDLLM_ERR_INVALID_ARG, "layer_step_noalloc: null cfg or step");
  if (!k_pool || !v_pool || !rope_cos || !rope_sin)
    return fail(FDLLM_ERR_INVALID_ARG, "layer_step_noalloc: null pool or RoPE table");
  if ((reinterpret_cast<uintptr_t>(k_pool) | reinterpret_cast<uintptr_t>(v_pool) |
       reinterpret_cast<uintptr_t>(rope_cos) | reinterpret_cast<uintptr_t>(rope_sin)) & 15)
    return fail(FDLLM_ERR_INVALID_ARG,
                "layer_step_noalloc: pools and RoPE tables must be 16-byte aligned");
  // The same configuration rules as fdllm_cache_create.
  const fdllm_cache_config& c = *cfg;
  if (c.n_layers <= 0 || c.n_heads <= 0 || c.head_dim <= 0 || c.page_size <= 0 ||
      c.num_pages <= 0 || c.max_position <= 0 || c.max_batch <= 0 || c.max_slots_per_seq <= 0)
    return fail(FDLLM_ERR_INVALID_ARG, "layer_step_noalloc: sizes must be positive");
  if (c.dtype != FDLLM_BF16 && c.dtype != FDLLM_F32)
    return fail(FDLLM_ERR_INVALID_ARG, "layer_step_noalloc: unknown dtype %d", c.dtype);
  if (c.head_dim % 2)
    return fail(FDLLM_ERR_INVALID_ARG, "layer_step_noalloc: head_dim must be even (RoPE pairs)");
  if (c.dtype == FDLLM_BF16 && c.head_dim != 128)
    return fail(FDLLM_ERR_UNSUPPORTED, "layer_step_noalloc: bf16 kernels serve head_dim 128 only");
  if (c.dtype == FDLLM_F32 && (c.head_dim > 128 || c.head_dim % 32))
    return fail(FDLLM_ERR_UNSUPPORTED,
                "layer_step_noalloc: fp32 kernel serves head_dim 32/64/96/128");
  if (c.max_batch > kMaxBatch)
    return fail(FDLLM_ERR_UNSUPPORTED, "layer_step_noalloc: max_batch > %d", kMaxBatch);
  if (c.dtype == FDLLM_BF16 && c.page_size != kBf16PageSize)
    return fail(FDLLM_ERR_UNSUPPORTED, "layer_step_noalloc: bf16 kernels gather %d-slot pages",
                kBf16PageSize);
  if ((long long)c.n_layers * c.num_pages * c.n_heads * c.page_size >= (1ll << 31))
    return fail(FDLLM_ERR_UNSUPPORTED, "layer_step_noalloc: pool has 2^31 or more slot rows");
  if (st->batch <= 0 || st->max_blocks_per_seq <= 0)
    return fail(FDLLM_ERR_INVALID_ARG,
                "layer_step_noalloc: batch and max_blocks_per_seq must be positive");
  // The fixed scratch bounds the mass partials: n_heads * batch * row length.
  if (attn_mass) {
    const long long need =
        (long long)c.n_heads * st->batch * st->max_blocks_per_seq * c.page_size;
    if (need > (long long)kNoAllocPartFloats)
      return fail(FDLLM_ERR_UNSUPPORTED,
                  "layer_step_noalloc: the attention-mass scratch needs %lld floats "
                  "(n_heads * batch * max_blocks_per_seq * page_size), more than the %zu that "
                  "fit in the library's fixed %zu-byte buffer; pass attn_mass = NULL or use "
                  "fdllm_layer_step",
                  need, kNoAllocPartFloats, kNoAllocScratchBytes);
  }

  void* scratch = nullptr;
  fdllm_status ss = noalloc_scratch(reinterpret_cast<cudaStream_t>(stream), &scratch);
  if (ss != FDLLM_OK) return ss;

  // A handle on the stack over the caller's memory and the fixed scratch;
  // fdllm_layer_step does the rest (checks, plan, launches).
  fdllm_cache h;
  memset(&h, 0, sizeof(h));
  h.cfg = c;
  h.k_pool = k_pool;
  h.v_pool = v_pool;
  if (c.dtype == FDLLM_BF16) {
    const uint64_t rows = (uint64_t)c.n_layers * c.num_pages * c.n_heads * c.page_size;
    if (!encode_bf16_2d(&h.tmap_k, k_pool, rows, (uint64_t)c.head_dim, (uint32_t)c.page_size) ||
        !encode_bf16_2d(&h.tmap_v, v_pool, rows, (uint64_t)c.head_dim, (uint32_t)c.page_size))
      return fail(FDLLM_ERR_CUDA, "layer_step_noalloc: cuTensorMapEncodeTiled failed for the pools");
  }
  cudaGetDevice(&h.device);
  h.rope_cos = const_cast<double*>(rope_cos);
  h.rope_sin = const_cast<double*>(rope_sin);
  h.mass_part = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + kNoAllocPartOffset);
  h.mass_part_floats = kNoAllocPartFloats;
  h.err = static_cast<int*>(scratch);

  fdllm_status s = fdllm_layer_step(&h, layer, st, x, wqkv, positions, block_table, view_mask, out,
                                    attn_mass, stream);
  if (s != FDLLM_OK || !st->validate) return s;
  // validate = 1: fdllm_layer_step has synchronised the stream; report and
  // clear what the kernels recorded in the error word.
  int w[4];
  cudaError_t e;
  if ((e = cudaMemcpy(w, h.err, sizeof(w), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "layer_step_noalloc: read error word");
  if (w[0] == 0) return FDLLM_OK;
  if ((e = cudaMemsetAsync(h.err, 0, sizeof(w), reinterpret_cast<cudaStream_t>(stream))) !=
      cudaSuccess)
    return cuda_fail(e, "layer_step_noalloc: clear error word");
  // The word is shared by every call on this device: what it holds may have
  // been recorded by an earlier call made with validate = 0.
  if (w[0] == kDevTimeout)
    return fail(FDLLM_ERR_TIMEOUT,
                "device: bounded wait timed out (site %d), in this call or an earlier "
                "validate = 0 call on this device",
                w[1]);
  return fail(FDLLM_ERR_DEVICE_BOUNDS,
              "device: metadata out of range (code %d, detail %d), in this call or an earlier "
              "validate = 0 call on this device",
              w[0], w[1]);
}

}  // extern "C"
