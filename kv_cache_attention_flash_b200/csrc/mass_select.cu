// Attention-mass reduction over heads and top-k tracking selection.
//
// "Flash-dLLM: I/O-Aware KV Caching and Parallel Decoding for Fast,
// Memory-Efficient Diffusion LLMs" (ai4snews summary), paragraph 2: only a
// fixed budget of the most-attended tokens is tracked and updated. The step
// kernels write each head's per-key probability sums; this file turns them
// into the per-sequence mass (mean over heads and rows, summed in a fixed
// head order so the result is reproducible bit for bit) and selects the k
// slots of largest mass.
#include <cstdint>

#include "fdllm_internal.h"

namespace fdllm {
namespace {

__global__ void mass_reduce_kernel(const __grid_constant__ StepPlan plan, const float* part,
                                   float* mass, int n_heads) {
  const int b = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= plan.row_stride) return;
  const int n = plan.cu_rows[b + 1] - plan.cu_rows[b];
  float s = 0.f;
  if (n > 0) {
    const size_t hs = (size_t)plan.batch * plan.row_stride;
    const float* p = part + (size_t)b * plan.row_stride + j;
    for (int h = 0; h < n_heads; ++h) s += p[h * hs];
    s *= 1.0f / (float)(n * n_heads);
  }
  mass[(size_t)b * plan.row_stride + j] = s;
}

// The same reduction four slots per thread, for row strides that are a
// multiple of 4 and a 16-byte aligned output; heads are summed in the same
// order, so both give the same bits.
__global__ void mass_reduce4_kernel(const __grid_constant__ StepPlan plan, const float* part,
                                    float* mass, int n_heads) {
  const int b = blockIdx.y;
  const int j = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (j >= plan.row_stride) return;
  const int n = plan.cu_rows[b + 1] - plan.cu_rows[b];
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  if (n > 0) {
    const size_t hs = (size_t)plan.batch * plan.row_stride;
    const float* p = part + (size_t)b * plan.row_stride + j;
    // 16 heads' loads in flight at a time, added in head order
    for (int h0 = 0; h0 < n_heads; h0 += 16) {
      float4 v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (h0 + u < n_heads) v[u] = __ldg(reinterpret_cast<const float4*>(p + (h0 + u) * hs));
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (h0 + u < n_heads) {
          s.x += v[u].x;
          s.y += v[u].y;
          s.z += v[u].z;
          s.w += v[u].w;
        }
    }
    const float sc = 1.0f / (float)(n * n_heads);
    s.x *= sc;
    s.y *= sc;
    s.z *= sc;
    s.w *= sc;
  }
  *reinterpret_cast<float4*>(mass + (size_t)b * plan.row_stride + j) = s;
}

// Order-preserving map of a float to an unsigned key (larger float, larger key).
__device__ __forceinline__ uint32_t fkey(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int SEL_THREADS = 1024;
constexpr int SEL_MAXK = 1024;
constexpr int SEL_MAXL = 65536;
constexpr int SEL_SMEM_KEYS = 5120;   // rows up to this length keep their keys on chip

// A candidate as one 64-bit word ordered like (key descending, slot
// ascending): key in the high half, the slot's complement in the low half.
// 0 marks "no candidate" (below every real one: slots are < 2^31).
__device__ __forceinline__ uint64_t cand_word(uint32_t key, int slot) {
  return ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)slot);
}

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ uint64_t shfl_u64(uint64_t v, int src) {
  const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)v, src);
  const uint32_t hi = __shfl_sync(0xffffffffu, (uint32_t)(v >> 32), src);
  return ((uint64_t)hi << 32) | lo;
}

// Bitonic sort across a warp, one word per lane: lane i ends with the i-th
// largest. Blocks of `size` lanes alternate direction until the last stage.
__device__ __forceinline__ uint64_t warp_sort_desc(uint64_t v, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint64_t o = shfl_xor_u64(v, stride);
      const bool keep_max = ((lane & stride) == 0) == ((lane & size) == 0);
      v = keep_max ? (v > o ? v : o) : (v < o ? v : o);
    }
  return v;
}

// The 32 largest of two descending warp lists: the elementwise maximum of
// one list and the other reversed is bitonic and holds them; a bitonic merge
// sorts it.
__device__ __forceinline__ uint64_t warp_merge_top(uint64_t a, uint64_t b, int lane) {
  const uint64_t br = shfl_u64(b, 31 - lane);
  uint64_t c = a > br ? a : br;
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) {
    const uint64_t o = shfl_xor_u64(c, stride);
    c = (lane & stride) == 0 ? (c > o ? c : o) : (c < o ? c : o);
  }
  return c;
}

// One CTA per sequence.
// k <= 32: each warp keeps the 32 largest candidate words of its chunks of
// 32 slots, sorted in registers (a chunk is sorted only when one of its
// words beats the warp's 32nd); the warps' lists are then merged pairwise.
// Larger k: exact radix select of the k-th largest key (4 passes of 8 bits),
// then the strictly larger keys plus the lowest-slot ties, then a bitonic
// sort by (key descending, slot ascending). Both give the same slots in the
// same order.
__global__ void __launch_bounds__(SEL_THREADS)
    select_kernel(const float* mass, const int32_t* seq_lens, int row_stride, int k,
                  const int32_t* exclude_cu, const int32_t* exclude_slots, int32_t* tracked) {
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const float* m = mass + (size_t)b * row_stride;
  int L = seq_lens[b];
  if (L < 0) L = 0;
  if (L > row_stride) L = row_stride;

  __shared__ uint32_t excl[SEL_MAXL / 32];
  __shared__ int hist[256];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;
  __shared__ int s_total;
  __shared__ int s_cnt;
  __shared__ int s_eqbase;
  __shared__ uint32_t sk[SEL_MAXK];
  __shared__ int ss[SEL_MAXK];
  __shared__ int warp_sums[SEL_THREADS / 32];
  __shared__ __align__(16) uint32_t skey[SEL_SMEM_KEYS];
  static_assert(SEL_THREADS * 8 <= SEL_SMEM_KEYS * 4, "warp lists fit in the key buffer");
  const bool fast = k <= 32;
  const bool staged = !fast && L <= SEL_SMEM_KEYS;
  if (staged)
    for (int j = tid; j < L; j += SEL_THREADS) skey[j] = fkey(__ldg(m + j));
  auto key_of = [&](int j) -> uint32_t { return staged ? skey[j] : fkey(__ldg(m + j)); };

  for (int i = tid; i < (L + 31) / 32; i += SEL_THREADS) excl[i] = 0u;
  __syncthreads();
  if (exclude_cu) {
    const int e0 = exclude_cu[b], e1 = exclude_cu[b + 1];
    for (int e = e0 + tid; e < e1; e += SEL_THREADS) {
      const int s = exclude_slots[e];
      if (s >= 0 && s < L) atomicOr(&excl[s >> 5], 1u << (s & 31));
    }
  }
  if (tid == 0) s_total = 0;
  __syncthreads();
  if (fast) {
    constexpr int NW = SEL_THREADS / 32;
    const int lane = tid & 31, warp = tid >> 5;
    uint64_t top = 0;
    for (int base = warp * 32; base < L; base += SEL_THREADS) {
      const int j = base + lane;
      uint64_t v = 0;
      if (j < L && !((excl[j >> 5] >> (j & 31)) & 1u)) v = cand_word(fkey(__ldg(m + j)), j);
      if (__ballot_sync(0xffffffffu, v > shfl_u64(top, 31)) == 0u) continue;
      top = warp_merge_top(top, warp_sort_desc(v, lane), lane);
    }
    uint64_t* lists = reinterpret_cast<uint64_t*>(skey);   // [NW][32], unused in this path
    lists[warp * 32 + lane] = top;
    __syncthreads();
#pragma unroll 1
    for (int half = NW / 2; half > 0; half >>= 1) {
      if (warp < half) {
        const uint64_t c = warp_merge_top(lists[warp * 32 + lane], lists[(warp + half) * 32 + lane],
                                          lane);
        lists[warp * 32 + lane] = c;
      }
      __syncthreads();
    }
    if (tid < k) {
      const uint64_t c = lists[tid];
      tracked[(size_t)b * k + tid] = c ? (int)(0xFFFFFFFFu - (uint32_t)c) : -1;
    }
    return;
  }
  // candidate count (one shared atomic per warp)
  {
    int c = 0;
    for (int j = tid; j < L; j += SEL_THREADS) c += ((excl[j >> 5] >> (j & 31)) & 1u) ? 0 : 1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if ((tid & 31) == 0 && c) atomicAdd(&s_total, c);
  }
  __syncthreads();
  const int total = s_total;
  const int want = total < k ? total : k;

  uint32_t prefix = 0, pmask = 0;
  int remaining = want;
  if (want > 0 && want < total) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += SEL_THREADS) hist[i] = 0;
      __syncthreads();
      for (int base = 0; base < L; base += SEL_THREADS) {
        const int j = base + tid;
        bool in = false;
        uint32_t dig = 0u;
        if (j < L && !((excl[j >> 5] >> (j & 31)) & 1u)) {
          const uint32_t key = key_of(j);
          in = (key & pmask) == prefix;
          dig = (key >> shift) & 255u;
        }
        // one shared atomic per distinct digit in the warp (keys cluster in
        // few digits, e.g. a shared exponent byte)
        const uint32_t act = __ballot_sync(0xffffffffu, in);
        if (in) {
          const uint32_t same = __match_any_sync(act, dig);
          if ((tid & 31) == __ffs(same) - 1) atomicAdd(&hist[dig], __popc(same));
        }
      }
      __syncthreads();
      if (tid < 32) {
        // the digit (scanning down from 255) at which the count of keys
        // above reaches `remaining`: lane l holds digits 255-8l .. 248-8l
        int c[8], sum = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          c[q] = hist[255 - 8 * tid - q];
          sum += c[q];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (tid >= o) incl += t;
        }
        const int ex = incl - sum;
        const uint32_t ball = __ballot_sync(0xffffffffu, ex < remaining && incl >= remaining);
        if (ball != 0u && tid == __ffs(ball) - 1) {
          int cum = ex, d = 248 - 8 * tid;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (cum + c[q] >= remaining) {
              d = 255 - 8 * tid - q;
              break;
            }
            cum += c[q];
          }
          s_prefix = prefix | ((uint32_t)d << shift);
          s_remaining = remaining - cum;
        }
      }
      __syncthreads();
      prefix = s_prefix;
      remaining = s_remaining;
      pmask |= 255u << shift;
      __syncthreads();
    }
  }
  // threshold key T = prefix (when want < total); take every key > T and the
  // `remaining` lowest slots with key == T.
  const bool all = (want == total);
  if (tid == 0) s_cnt = 0;
  __syncthreads();
  for (int j = tid; j < L; j += SEL_THREADS) {
    if ((excl[j >> 5] >> (j & 31)) & 1u) continue;
    const uint32_t key = key_of(j);
    if (all || key > prefix) {
      const int p = atomicAdd(&s_cnt, 1);
      sk[p] = key;
      ss[p] = j;
    }
  }
  __syncthreads();
  if (!all && remaining > 0) {
    // ties at the threshold, lowest slots first: block-wide scan in slot order
    if (tid == 0) s_eqbase = 0;
    __syncthreads();
    for (int base = 0; base < L; base += SEL_THREADS) {
      const int j = base + tid;
      int f = 0;
      if (j < L && !((excl[j >> 5] >> (j & 31)) & 1u) && key_of(j) == prefix) f = 1;
      // inclusive scan of f across the block
      int v = f;
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if ((tid & 31) >= o) v += t;
      }
      if ((tid & 31) == 31) warp_sums[tid >> 5] = v;
      __syncthreads();
      if (tid < 32) {
        constexpr int NW = SEL_THREADS / 32;
        int w = tid < NW ? warp_sums[tid] : 0;
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, w, o);
          if (tid >= o) w += t;
        }
        if (tid < NW) warp_sums[tid] = w;
      }
      __syncthreads();
      const int excl_before = (tid >= 32 ? warp_sums[(tid >> 5) - 1] : 0) + v - f;
      const int rank = s_eqbase + excl_before;
      if (f && rank < remaining) {
        const int p = (want - remaining) + rank;
        sk[p] = prefix;
        ss[p] = j;
      }
      __syncthreads();
      if (tid == 0) s_eqbase += warp_sums[SEL_THREADS / 32 - 1];
      __syncthreads();
      if (s_eqbase >= remaining) break;
    }
  }
  __syncthreads();
  // pad and sort by (key desc, slot asc)
  int P2 = 1;
  while (P2 < want) P2 <<= 1;
  for (int i = want + tid; i < P2; i += SEL_THREADS) {
    sk[i] = 0u;
    ss[i] = 0x7fffffff;
  }
  __syncthreads();
  for (int size = 2; size <= P2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < P2; i += SEL_THREADS) {
        const int jx = i ^ stride;
        if (jx > i) {
          const bool up = (i & size) == 0;   // "up" = descending by (key, -slot)
          const uint32_t ka = sk[i], kb = sk[jx];
          const int sa = ss[i], sb = ss[jx];
          const bool a_first = (ka > kb) || (ka == kb && sa < sb);
          if (up ? !a_first : a_first) {
            sk[i] = kb;
            sk[jx] = ka;
            ss[i] = sb;
            ss[jx] = sa;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < k; i += SEL_THREADS)
    tracked[(size_t)b * k + i] = (i < want) ? ss[i] : -1;
}

}  // namespace

cudaError_t launch_mass_reduce(const StepPlan& plan, const float* part, float* mass, int n_heads,
                               cudaStream_t stream) {
  if (plan.row_stride % 4 == 0 && (reinterpret_cast<uintptr_t>(mass) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(part) & 15) == 0) {
    dim3 grid((plan.row_stride / 4 + 63) / 64, plan.batch);
    mass_reduce4_kernel<<<grid, 64, 0, stream>>>(plan, part, mass, n_heads);
  } else {
    dim3 grid((plan.row_stride + 255) / 256, plan.batch);
    mass_reduce_kernel<<<grid, 256, 0, stream>>>(plan, part, mass, n_heads);
  }
  return cudaGetLastError();
}

cudaError_t launch_select_tracked(const float* mass, const int32_t* seq_lens, int batch,
                                  int row_stride, int k, const int32_t* exclude_cu,
                                  const int32_t* exclude_slots, int32_t* tracked,
                                  cudaStream_t stream) {
  select_kernel<<<batch, SEL_THREADS, 0, stream>>>(mass, seq_lens, row_stride, k, exclude_cu,
                                                   exclude_slots, tracked);
  return cudaGetLastError();
}

}  // namespace fdllm
