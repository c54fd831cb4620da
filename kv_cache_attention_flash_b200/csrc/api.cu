// Host side of the C ABI declared in include/fdllm.h: argument checks, the
// row-group plan, TMA descriptors, kernel launches and error reporting.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <set>
#include <string>
#include <vector>

#include "fdllm.h"
#include "fdllm_internal.h"

using namespace fdllm;

namespace {

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
// {64, 64, 2, 3, 1} is one head's q, k and v columns for 64 K rows, written
// to shared memory as six 8 KB [64 rows][128 B] sub-boxes (128-byte swizzle).
bool encode_wqkv_5d(CUtensorMap* map, const void* base, uint64_t hidden, uint64_t n_heads,
                    uint64_t head_dim) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[5] = {64, hidden, head_dim / 64, 3, n_heads};
  cuuint64_t strides[4] = {3 * hidden * 2, 128, hidden * 2, head_dim * 2};
  cuuint32_t box[5] = {64, 64, (cuuint32_t)(head_dim / 64), 3, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

struct fdllm_cache {
  fdllm_cache_config cfg;
  CUtensorMap tmap_k;   // pools viewed as [rows = layer/page/head/slot][head_dim] (bf16)
  CUtensorMap tmap_v;
  void* k_pool;
  void* v_pool;
  int device;
  float* rope_cos;
  float* rope_sin;
  float* mass_part;
  size_t mass_part_floats;
  int* err;
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

  // RoPE tables in double on the host, stored fp32: angle p * theta^(-2i/D).
  const int half = c.head_dim / 2;
  const size_t nt = (size_t)c.max_position * half;
  std::vector<float> cs(nt), sn(nt);
  for (int p = 0; p < c.max_position; ++p)
    for (int i = 0; i < half; ++i) {
      const double inv = std::pow((double)c.rope_theta, -2.0 * i / c.head_dim);
      const double phi = (double)p * inv;
      cs[(size_t)p * half + i] = (float)std::cos(phi);
      sn[(size_t)p * half + i] = (float)std::sin(phi);
    }
  h->mass_part_floats = (size_t)c.n_heads * c.max_batch * c.max_slots_per_seq;
  cudaError_t e;
  if ((e = cudaMalloc(&h->rope_cos, nt * sizeof(float))) != cudaSuccess ||
      (e = cudaMalloc(&h->rope_sin, nt * sizeof(float))) != cudaSuccess ||
      (e = cudaMalloc(&h->mass_part, h->mass_part_floats * sizeof(float))) != cudaSuccess ||
      (e = cudaMalloc(&h->err, 4 * sizeof(int))) != cudaSuccess) {
    fdllm_cache_destroy(h);
    return cuda_fail(e, "cache_create: cudaMalloc");
  }
  if ((e = cudaMemcpyAsync(h->rope_cos, cs.data(), nt * sizeof(float), cudaMemcpyHostToDevice,
                           st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(h->rope_sin, sn.data(), nt * sizeof(float), cudaMemcpyHostToDevice,
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
                              const int32_t* block_table, const int8_t* view_mask, float* out,
                              float* attn_mass, void* stream) {
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
      if (!encode_wqkv_5d(&tw, wqkv, (uint64_t)H, (uint64_t)c.n_heads, (uint64_t)c.head_dim))
        return fail(FDLLM_ERR_CUDA, "layer_step: cuTensorMapEncodeTiled failed (wqkv)");
      e = launch_step_bf16(plan, a, txp, &tw, &h->tmap_k, &h->tmap_v, s);
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

fdllm_status fdllm_check(fdllm_cache* h, void* stream) {
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
                                      const float* rope_cos, const float* rope_sin, int32_t layer,
                                      const fdllm_step* st, const void* x, const void* wqkv,
                                      const int32_t* positions, const int32_t* block_table,
                                      const int8_t* view_mask, float* out, float* attn_mass,
                                      void* stream) {
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
  h.rope_cos = const_cast<float*>(rope_cos);
  h.rope_sin = const_cast<float*>(rope_sin);
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
  if (w[0] == kDevTimeout)
    return fail(FDLLM_ERR_TIMEOUT, "device: bounded wait timed out (site %d)", w[1]);
  return fail(FDLLM_ERR_DEVICE_BOUNDS, "device: metadata out of range (code %d, detail %d)", w[0],
              w[1]);
}

}  // extern "C"
