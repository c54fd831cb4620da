// Flash-Verify acceptance: the mask view's prediction and confidence at every
// block position, and each sequence's accepted prefix.
//
// "Flash-dLLM: I/O-Aware KV Caching and Parallel Decoding for Fast,
// Memory-Efficient Diffusion LLMs" (ai4snews summary), paragraph 3: a
// position is accepted only when the draft view and the mask view agree and
// the mask view's confidence exceeds a threshold; acceptance runs in causal
// order and stops at the first position that fails.
//
// The logits are read once (HBM-bound): one CTA per row streams the
// vocabulary with 16-byte loads, each thread keeping the running largest
// logit (compared as stored, so ties go to the lowest token id), its index
// and the sum of 2^((logit - max) * log2 e); the partial triples are merged
// across the block. A second, one-thread-per-sequence launch scans the
// sequence's positions in order.
#include <cuda_bf16.h>

#include <cstdint>

#include "fdllm_internal.h"
#include "ptx.cuh"

namespace fdllm {
namespace {

constexpr int VT = 512;                 // threads per row
constexpr float kLog2e = 1.4426950408889634f;

struct Acc {
  float m;     // largest logit seen
  int idx;     // its lowest index
  float s;     // sum of 2^((l - m) * log2 e) over the logits seen
};

__device__ __forceinline__ void push(Acc& a, float l, int i) {
  if (l > a.m) {
    a.s = a.s * ptx::ex2((a.m - l) * kLog2e) + 1.f;   // a.m = -inf: 0 * 0 + 1
    a.m = l;
    a.idx = i;
  } else if (l > -INFINITY) {
    a.s += ptx::ex2((l - a.m) * kLog2e);
  }
}

// b into a: the larger maximum wins (equal maxima: the lower index).
__device__ __forceinline__ void merge(Acc& a, Acc b) {
  if (b.m > a.m || (b.m == a.m && b.idx < a.idx)) {
    const Acc t = a;
    a = b;
    b = t;
  }
  if (b.m > -INFINITY) a.s += b.s * ptx::ex2((b.m - a.m) * kLog2e);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// N consecutive logits (indices e0 .. e0+N-1) at once: their maximum first
// (at most one rescale of the running sum), then N independent exponentials
// added as a tree, so a thread keeps N exponentials in flight.
template <int N>
__device__ __forceinline__ void push_n(Acc& a, const float* v, int e0) {
  float lm = v[0];
  int li = 0;
#pragma unroll
  for (int i = 1; i < N; ++i)
    if (v[i] > lm) {
      lm = v[i];
      li = i;
    }
  if (lm > a.m) {
    a.s *= ptx::ex2((a.m - lm) * kLog2e);   // a.m = -inf: 0
    a.m = lm;
    a.idx = e0 + li;
  }
  if (a.m == -INFINITY) return;             // nothing finite seen yet
  const float mc = a.m * kLog2e;
  float t[N];
#pragma unroll
  for (int i = 0; i < N; ++i) t[i] = ptx::ex2(fmaf(v[i], kLog2e, -mc));
#pragma unroll
  for (int w = N / 2; w > 0; w /= 2)
#pragma unroll
    for (int i = 0; i < w; ++i) t[i] += t[i + w];
  a.s += t[0];
}

__device__ __forceinline__ void push_vec(Acc& a, const uint4& w, int e0, bool bf16) {
  const uint32_t q[4] = {w.x, w.y, w.z, w.w};
  if (bf16) {
    float v[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = bf16_lo(q[k]);
      v[2 * k + 1] = bf16_hi(q[k]);
    }
    push_n<8>(a, v, e0);
  } else {
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = __uint_as_float(q[k]);
    push_n<4>(a, v, e0);
  }
}

template <bool kBf16>
__global__ void __launch_bounds__(VT) verify_rows_kernel(const void* logits, int vocab,
                                                         int32_t* pred, float* conf) {
  const int r = blockIdx.x;
  const int tid = threadIdx.x;
  constexpr int EPV = kBf16 ? 8 : 4;    // elements per 16-byte load
  const size_t row_bytes = (size_t)vocab * (kBf16 ? 2 : 4);
  const uint8_t* row = reinterpret_cast<const uint8_t*>(logits) + (size_t)r * row_bytes;
  Acc a{-INFINITY, 0x7fffffff, 0.f};
  const bool vec = (row_bytes % 16 == 0) && ((reinterpret_cast<uintptr_t>(row) & 15) == 0);
  int done = 0;
  if (vec) {
    const uint4* v4 = reinterpret_cast<const uint4*>(row);
    const int nvec = vocab / EPV;
    constexpr int U = 8;                  // loads in flight per thread
    int i = tid;
    for (; i + (U - 1) * VT < nvec; i += U * VT) {
      uint4 w[U];
#pragma unroll
      for (int u = 0; u < U; ++u) w[u] = __ldg(v4 + i + u * VT);
#pragma unroll
      for (int u = 0; u < U; ++u) push_vec(a, w[u], (i + u * VT) * EPV, kBf16);
    }
    for (; i < nvec; i += VT) push_vec(a, __ldg(v4 + i), i * EPV, kBf16);
    done = nvec * EPV;
  }
  // the rest one element at a time (all of an unaligned row)
  for (int e = done + tid; e < vocab; e += VT) {
    float l;
    if (kBf16) {
      const uint16_t u = reinterpret_cast<const uint16_t*>(row)[e];
      l = __uint_as_float((uint32_t)u << 16);
    } else {
      l = reinterpret_cast<const float*>(row)[e];
    }
    push(a, l, e);
  }
  // block merge: warps by shuffle, then the warp results
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Acc b;
    b.m = __shfl_xor_sync(0xffffffffu, a.m, o);
    b.idx = __shfl_xor_sync(0xffffffffu, a.idx, o);
    b.s = __shfl_xor_sync(0xffffffffu, a.s, o);
    merge(a, b);
  }
  __shared__ Acc wacc[VT / 32];
  if ((tid & 31) == 0) wacc[tid >> 5] = a;
  __syncthreads();
  if (tid == 0) {
    Acc t = wacc[0];
    for (int w = 1; w < VT / 32; ++w) merge(t, wacc[w]);
    pred[r] = t.m > -INFINITY ? t.idx : 0;
    conf[r] = t.s > 0.f ? 1.f / t.s : 0.f;
  }
}

__global__ void verify_scan_kernel(const int32_t* cu_rows, int batch, int rows,
                                   const int32_t* draft, const int32_t* pred, const float* conf,
                                   float tau, int32_t* n_accepted) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch) return;
  int r0 = cu_rows[b], r1 = cu_rows[b + 1];
  r0 = r0 < 0 ? 0 : (r0 > rows ? rows : r0);
  r1 = r1 < r0 ? r0 : (r1 > rows ? rows : r1);
  int n = 0;
  for (int i = r0; i < r1; ++i) {
    if (pred[i] == draft[i] && conf[i] > tau) ++n;
    else break;
  }
  n_accepted[b] = n;
}

}  // namespace

cudaError_t launch_verify_accept(const void* logits, bool bf16, int rows, int vocab,
                                 const int32_t* cu_rows, int batch, const int32_t* draft,
                                 float tau, int32_t* pred, float* conf, int32_t* n_accepted,
                                 cudaStream_t stream) {
  if (rows > 0) {
    if (bf16)
      verify_rows_kernel<true><<<rows, VT, 0, stream>>>(logits, vocab, pred, conf);
    else
      verify_rows_kernel<false><<<rows, VT, 0, stream>>>(logits, vocab, pred, conf);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  verify_scan_kernel<<<(batch + 127) / 128, 128, 0, stream>>>(cu_rows, batch, rows, draft, pred,
                                                              conf, tau, n_accepted);
  return cudaGetLastError();
}

}  // namespace fdllm
