// Plain fp32 kernels on CUDA cores for small, non-FP8 shapes (e.g. 4 indexer
// heads of 32 dims, 8 query heads over 64-dim keys). Same definitions as the
// tensor-core path:
//   indexer  I[t,s] = sum_j w[t,j] * max(0, q_I[t,j] . k_I[s])   (jdon.com
//            "DeepSeek-V3.2-Exp", lightning-indexer paragraph)
//   attention over the selected rows with key = whole row, value = first Dv dims
//            (openi.cn "DeepSeek-V3.2", MLA-in-MQA-mode item).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int kIdxThreads = 128;

__global__ void __launch_bounds__(kIdxThreads)
    indexer_f32_kernel(const float *__restrict__ q, const float *__restrict__ kI, const float *__restrict__ w,
                       int H_I, int d_I, Layout L, float *__restrict__ scores, long long ld, ErrCtx e) {
  extern __shared__ float sq[];  // [H_I*d_I] query heads, then [H_I] weights
  pdl_prologue();
  const int t = blockIdx.y;
  const RowPos rp = row_position(L, t);
  const int s0 = blockIdx.x * kIdxThreads;
  if (s0 > rp.pos) return;
  if (rp.len > L.n_max) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_error(e, DEV_BOUNDS, 0x200);
    return;
  }
  const int nq = H_I * d_I;
  for (int i = threadIdx.x; i < nq; i += kIdxThreads) sq[i] = q[(long long)t * nq + i];
  for (int i = threadIdx.x; i < H_I; i += kIdxThreads) sq[nq + i] = w[(long long)t * H_I + i];
  __syncthreads();
  const int s = s0 + threadIdx.x;
  if (s > rp.pos) return;
  const float *krow = kI + ((long long)rp.b * L.n_max + s) * d_I;
  float acc = 0.f;
  for (int j = 0; j < H_I; ++j) {
    const float *qj = sq + j * d_I;
    float dot = 0.f;
    for (int d = 0; d < d_I; ++d) dot = fmaf(qj[d], __ldg(krow + d), dot);
    acc = fmaf(sq[nq + j], fmaxf(dot, 0.f), acc);
  }
  scores[(long long)t * ld + s] = acc;
}

constexpr int kAttnThreads = 256;

__device__ __forceinline__ float block_reduce(float v, float *red, bool is_max) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float o = __shfl_xor_sync(0xFFFFFFFFu, v, off);
    v = is_max ? fmaxf(v, o) : v + o;
  }
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kAttnThreads / 32; ++i) r = is_max ? fmaxf(r, red[i]) : r + red[i];
  return r;
}

// One CTA per (query row, head). z_i for the selected rows is kept in shared memory.
__global__ void __launch_bounds__(kAttnThreads)
    attn_f32_kernel(const float *__restrict__ q, const float *__restrict__ kv, int H, int Dk, int Dv, float scale,
                    const int *__restrict__ idx, int k, Layout L, float *__restrict__ out, float *__restrict__ lse,
                    ErrCtx e) {
  extern __shared__ float smf[];
  float *z = smf;                                      // [k]
  long long *rows = reinterpret_cast<long long *>(smf + ((k + 1) & ~1));  // [k]
  __shared__ float red[kAttnThreads / 32];
  pdl_prologue();
  const int t = blockIdx.x, h = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const RowPos rp = row_position(L, t);
  const float *qh = q + ((long long)t * H + h) * Dk;

  for (int i = threadIdx.x; i < k; i += kAttnThreads) {
    const int s = idx[(long long)t * k + i];
    long long r = -1;
    if (s >= 0) {
      if (s > rp.pos || rp.len > L.n_max) raise_error(e, DEV_BOUNDS, 0x300);
      else r = (long long)rp.b * L.n_max + s;
    } else if (s != -1) {
      raise_error(e, DEV_BOUNDS, 0x301);
    }
    rows[i] = r;
  }
  __syncthreads();
  // scores: one warp per selected row
  for (int i = warp; i < k; i += kAttnThreads / 32) {
    const long long r = rows[i];
    float dot = 0.f;
    if (r >= 0) {
      const float *kr = kv + r * Dk;
      for (int d = lane; d < Dk; d += 32) dot = fmaf(qh[d], kr[d], dot);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, off);
    if (lane == 0) z[i] = r >= 0 ? dot * scale : -INFINITY;
  }
  __syncthreads();
  float m = -INFINITY;
  for (int i = threadIdx.x; i < k; i += kAttnThreads) m = fmaxf(m, z[i]);
  m = block_reduce(m, red, true);
  float* orow = out + ((long long)t * H + h) * Dv;
  if (m == -INFINITY) {  // nothing selected
    for (int d = threadIdx.x; d < Dv; d += kAttnThreads) orow[d] = 0.f;
    if (lse && threadIdx.x == 0) lse[(long long)t * H + h] = -INFINITY;
    return;
  }
  float sum = 0.f;
  for (int i = threadIdx.x; i < k; i += kAttnThreads) {
    const float p = expf(z[i] - m);
    z[i] = p;
    sum += p;
  }
  sum = block_reduce(sum, red, false);
  const float inv = 1.f / sum;
  for (int d = threadIdx.x; d < Dv; d += kAttnThreads) {
    float acc = 0.f;
    for (int i = 0; i < k; ++i) {
      const long long r = rows[i];
      if (r >= 0) acc = fmaf(z[i], kv[r * Dk + d], acc);
    }
    orow[d] = acc * inv;
  }
  if (lse && threadIdx.x == 0) lse[(long long)t * H + h] = m + logf(sum);
}

}  // namespace

cudaError_t launch_indexer_f32(const float *q, const float *kI, const float *w, int T, int H_I, int d_I,
                               const Layout &L, float *scores, long long ld, const ErrCtx &e, cudaStream_t stream) {
  const size_t smem = (size_t)(H_I * d_I + H_I) * sizeof(float);
  cudaError_t err = cudaFuncSetAttribute(indexer_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((unsigned)((L.n_max + kIdxThreads - 1) / kIdxThreads), (unsigned)T);
  return launch_kernel(indexer_f32_kernel, grid, dim3(kIdxThreads), smem, stream, 0, q, kI, w, H_I, d_I, L, scores,
                       ld, e);
}

cudaError_t launch_attn_f32(const float *q, const float *kv, int T, int H, int Dk, int Dv, float scale,
                            const int *idx, int k, const Layout &L, float *out, float *lse, const ErrCtx &e,
                            cudaStream_t stream) {
  const size_t smem = (size_t)((k + 1) & ~1) * sizeof(float) + (size_t)k * sizeof(long long);
  cudaError_t err = cudaFuncSetAttribute(attn_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((unsigned)T, (unsigned)H);
  return launch_kernel(attn_f32_kernel, grid, dim3(kAttnThreads), smem, stream, 0, q, kv, H, Dk, Dv, scale, idx, k, L,
                       out, lse, e);
}

}  // namespace dsa
