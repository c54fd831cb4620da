// Flash-Cache layer step for fp32 caches (CUDA cores, fp32 arithmetic).
//
// Same contract as the bf16 kernel ("Flash-dLLM: I/O-Aware KV Caching and
// Parallel Decoding for Fast, Memory-Efficient Diffusion LLMs", ai4snews
// summary, paragraphs 1-3), for the fp32 layer shape: the projection, RoPE
// and cache write of each sequence's rows happen in one CTA that then attends
// over that sequence's pages. fp32 inputs keep full fp32 products here
// (tensor cores would round them to tf32). One CTA per (sequence, head);
// head_dim <= 128, at most 128 rows per sequence.
#include "fdllm_internal.h"

namespace fdllm {
namespace {

constexpr int NT = 256;
constexpr int RB = 16;        // rows per projection block
constexpr int KB = 32;        // K per projection tile
constexpr int MAXD = 128;

__device__ __forceinline__ void set_err(int* err, int code, int detail) {
  if (atomicCAS(err, 0, code) == 0) err[1] = detail;
}

__global__ void __launch_bounds__(NT)
    step_f32_kernel(const __grid_constant__ StepPlan plan, const __grid_constant__ StepArgs a) {
  const int b = blockIdx.x;
  const int h = blockIdx.y;
  const int r0 = plan.cu_rows[b];
  const int n = plan.cu_rows[b + 1] - r0;
  if (n == 0) return;
  const int L = plan.seq_lens[b];
  const int D = a.head_dim;
  const int H = a.hidden;
  const int ps = a.page_size;
  const int C3 = 3 * D;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* x = reinterpret_cast<const float*>(a.x);
  const float* w = reinterpret_cast<const float*>(a.wqkv);
  float* kpool = reinterpret_cast<float*>(a.k_pool);
  float* vpool = reinterpret_cast<float*>(a.v_pool);
  const int* bt = a.block_table + (size_t)b * plan.max_blocks;
  const size_t layer_base = (size_t)plan.layer * a.num_pages * a.n_heads * ps * D;

  extern __shared__ float dyn[];
  float (*xs)[KB] = reinterpret_cast<float (*)[KB]>(dyn);            // [RB][KB]
  float* ws = dyn + RB * KB;                                          // [KB][3D]
  float* tmp = ws + KB * C3;                                          // [RB][3D]
  float* qs = tmp + RB * C3;                                          // [128][D]
  __shared__ int rpos[128], rslot[128], rpage[128], rview[128];
  __shared__ int xrow[128];
  __shared__ float pbuf[8][32];
  __shared__ int nxs;

  // row metadata
  for (int i = tid; i < n; i += NT) {
    const int gr = r0 + i;
    const int pos = a.positions[gr];
    const int slot = a.slots ? a.slots[gr] : pos;
    int page = -1;
    if (pos < 0 || pos >= a.max_position) {
      set_err(a.err, kDevBadPosition, gr);
    } else if (slot < 0 || slot >= plan.row_stride) {
      set_err(a.err, kDevBadSlot, gr);
    } else {
      page = bt[slot / ps];
      if (page < 0 || page >= a.num_pages) {
        set_err(a.err, kDevBadPage, gr);
        page = -1;
      }
    }
    rpos[i] = pos;
    rslot[i] = slot;
    rpage[i] = page;
    rview[i] = a.view ? (int)a.view[gr] : 0;
  }
  __syncthreads();

  // ---- projection + RoPE + cache write, 16 rows at a time
  for (int rb = 0; rb < n; rb += RB) {
    const int nr = min(RB, n - rb);
    float acc[RB][2];
#pragma unroll
    for (int r = 0; r < RB; ++r) acc[r][0] = acc[r][1] = 0.f;
    for (int k0 = 0; k0 < H; k0 += KB) {
      for (int e = tid; e < RB * KB; e += NT) {
        const int r = e / KB, k = e % KB;
        xs[r][k] = (r < nr && k0 + k < H) ? x[(size_t)(r0 + rb + r) * H + k0 + k] : 0.f;
      }
      for (int e = tid; e < KB * C3; e += NT) {
        const int k = e / C3, c = e % C3;
        const int blk = c / D, dd = c % D;
        ws[k * C3 + c] = (k0 + k < H) ? w[(size_t)(k0 + k) * 3 * H + blk * H + h * D + dd] : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = tid + cc * NT;
        if (c < C3) {
          for (int k = 0; k < KB; ++k) {
            const float wv = ws[k * C3 + c];
#pragma unroll
            for (int r = 0; r < RB; ++r) acc[r][cc] = fmaf(xs[r][k], wv, acc[r][cc]);
          }
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int c = tid + cc * NT;
      if (c < C3)
        for (int r = 0; r < RB; ++r) tmp[r * C3 + c] = acc[r][cc];
    }
    __syncthreads();
    const int half = D / 2;
    for (int e = tid; e < nr * half; e += NT) {
      const int r = e / half, i = e % half;
      const int lr = rb + r;
      const bool ok = rpage[lr] >= 0;
      const int pos = ok ? rpos[lr] : 0;
      // rotation in double from the double tables, rounded to fp32 once
      const double cs = a.rope_cos[(size_t)pos * half + i];
      const double sn = a.rope_sin[(size_t)pos * half + i];
      const float* tr = tmp + r * C3;
      const double q1 = tr[i], q2 = tr[i + half];
      const double k1 = tr[D + i], k2 = tr[D + i + half];
      qs[lr * D + i] = ok ? (float)fma(q1, cs, -q2 * sn) : 0.f;
      qs[lr * D + i + half] = ok ? (float)fma(q2, cs, q1 * sn) : 0.f;
      if (ok) {
        const size_t off = layer_base + ((size_t)rpage[lr] * a.n_heads + h) * ps * D +
                           (size_t)(rslot[lr] % ps) * D;
        kpool[off + i] = (float)fma(k1, cs, -k2 * sn);
        kpool[off + i + half] = (float)fma(k2, cs, k1 * sn);
        vpool[off + i] = tr[2 * D + i];
        vpool[off + i + half] = tr[2 * D + i + half];
      }
    }
    __syncthreads();
  }

  // ---- attention: view rows' fresh slots follow the context keys
  if (tid == 0) {
    int nx = 0;
    for (int r = 0; r < n; ++r)
      if (rview[r] != 0) xrow[nx++] = r;
    nxs = nx;
  }
  float* part = a.mass_part ? a.mass_part + ((size_t)h * plan.batch + b) * plan.row_stride : nullptr;
  if (part)
    for (int j = tid; j < plan.row_stride; j += NT) part[j] = 0.f;
  __syncthreads();
  const int nk = L + nxs;
  const float scale = rsqrtf((float)D);
  const float* kp = kpool;
  const float* vp = vpool;

  for (int rbase = 0; rbase < n; rbase += 8) {
    const int r = rbase + warp;
    const bool rv = r < n;
    const int rview_r = rv ? rview[r] : 0;
    const int rpos_r = rv ? rpos[r] : 0;
    float m = -INFINITY, l = 0.f;
    float o[MAXD / 32];
#pragma unroll
    for (int u = 0; u < MAXD / 32; ++u) o[u] = 0.f;
    for (int pass = 0; pass < 2; ++pass) {
      float lse = 0.f;
      if (pass == 1) {
        for (int off = 16; off > 0; off >>= 1) {
          const float mo = __shfl_xor_sync(0xffffffffu, m, off);
          const float lo = __shfl_xor_sync(0xffffffffu, l, off);
          const float mn = fmaxf(m, mo);
          l = (mn == -INFINITY) ? 0.f : l * expf(m - mn) + lo * expf(mo - mn);
          m = mn;
        }
        lse = (l > 0.f) ? m + logf(l) : INFINITY;
      }
      for (int c0 = 0; c0 < nk; c0 += 32) {
        const int j = c0 + lane;
        bool vis = false;
        size_t off = 0;
        if (rv && j < nk) {
          int slot, page;
          if (j < L) {
            slot = j;
            page = bt[j / ps];
            vis = page >= 0 && page < a.num_pages;
            if (!vis) set_err(a.err, kDevBadPage, -1 - j);
          } else {
            const int xr = xrow[j - L];
            slot = rslot[xr];
            page = rpage[xr];
            vis = page >= 0 && rview_r != 0 && rview[xr] == rview_r && rpos[xr] <= rpos_r;
          }
          if (vis)
            off = layer_base + ((size_t)page * a.n_heads + h) * ps * D + (size_t)(slot % ps) * D;
        }
        // q . k over D (a multiple of 32): 16-byte loads of the key row,
        // several in flight (keys of the 32 lanes are different rows)
        float s = 0.f;
        if (vis) {
          const float4* k4 = reinterpret_cast<const float4*>(kp + off);
          const float4* q4 = reinterpret_cast<const float4*>(qs + r * D);
          float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
          for (int d4 = 0; d4 < D / 4; ++d4) {
            const float4 kv = __ldg(k4 + d4);
            const float4 qv = q4[d4];
            s4[d4 & 3] = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, s4[d4 & 3]))));
          }
          s = ((s4[0] + s4[1]) + (s4[2] + s4[3])) * scale;
        }
        if (pass == 0) {
          if (vis) {
            if (s > m) {
              l = l * expf(m - s) + 1.f;
              m = s;
            } else {
              l += expf(s - m);
            }
          }
        } else {
          const float p = vis ? expf(s - lse) : 0.f;
#pragma unroll 4
          for (int t = 0; t < 32; ++t) {
            const float pt = __shfl_sync(0xffffffffu, p, t);
            const size_t offt = __shfl_sync(0xffffffffu, off, t);
            if (pt != 0.f) {
#pragma unroll
              for (int u = 0; u < MAXD / 32; ++u)
                if (u < D / 32) o[u] = fmaf(pt, __ldg(vp + offt + u * 32 + lane), o[u]);
            }
          }
          if (part) {
            pbuf[warp][lane] = p;
            __syncthreads();
            if (tid < 32 && c0 + tid < nk) {
              float sum = 0.f;
              for (int w2 = 0; w2 < 8; ++w2) sum += pbuf[w2][tid];
              const int jj = c0 + tid;
              const int slot = (jj < L) ? jj : rslot[xrow[jj - L]];
              part[slot] += sum;
            }
            __syncthreads();
          }
        }
      }
    }
    if (rv)
      for (int u = 0; u < D / 32; ++u)
        static_cast<float*>(a.out)[(size_t)(r0 + r) * H + h * D + u * 32 + lane] = o[u];
  }
}

}  // namespace

size_t step_f32_smem_bytes(int head_dim) {
  return sizeof(float) * (size_t)(RB * KB + KB * 3 * head_dim + RB * 3 * head_dim + 128 * head_dim);
}

cudaError_t launch_step_f32(const StepPlan& plan, const StepArgs& a, cudaStream_t stream) {
  const size_t smem = step_f32_smem_bytes(a.head_dim);
  // opt in once per device, for the largest head_dim served
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = opt_in_smem(reinterpret_cast<const void*>(step_f32_kernel),
                              (int)step_f32_smem_bytes(MAXD), attr_done);
  if (e != cudaSuccess) return e;
  dim3 grid(plan.batch, a.n_heads);
  step_f32_kernel<<<grid, NT, smem, stream>>>(plan, a);
  return cudaGetLastError();
}

}  // namespace fdllm
