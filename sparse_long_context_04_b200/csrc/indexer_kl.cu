// Indexer loss on the selected set (sparse stage) and its gradient.
//
// jdon.com "DeepSeek-V3.2-Exp": warm-up paragraph (the indexer learns to copy how
// the main attention distributes its attention, through a KL-divergence loss) and
// sparse-training paragraph (indexer and main model trained together with
// separated gradients). For query row t with selected set S_t:
//   target  p(s) = (1/H) sum_h exp(z_h(s) - lse_h),   z_h(s) = scale * q[t,h] . kv[s]
//   indexer r(s) = exp(I[t,s] - LSE_I),  LSE_I = log sum_{s in S_t} exp(I[t,s])
//   loss_t = sum_s p(s) (log p(s) - log r(s)),   grad[t, j] = r(s_j) - p(s_j)
// with lse_h the row's attention log-sum-exp per head (as the attention call
// returns it), so p is the heads' mean attention over S_t.
//
// First path on the CUDA cores: one CTA per (row, 32 selected slots). The row's
// 128 x 576 bf16 query (rows padded to an odd number of words, so that the 32
// head lanes of a warp hit 32 banks) and the chunk's 32 latent rows sit in shared
// memory; thread (head, half) accumulates 16 key dot products in fp32.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int kH = 128, kDk = 576;
constexpr int kKeysPerCta = 32;
constexpr int kThreads = 256;                     // (head, half of the keys)
constexpr int kQStride = kDk + 2;                 // bf16 per padded query row: 289 words (odd)
constexpr int kSmem = kH * kQStride * 2 + kKeysPerCta * kDk * 2 + 16;

struct KlParams {
  const __nv_bfloat16 *q;    // [T][128][576]
  const __nv_bfloat16 *kv;   // rows of 576
  const int *idx;            // [T][k]
  int k;
  const float *lse;          // [T][128]
  const float *scores;       // [T][ld]
  long long ld;
  float scale;
  float *loss;               // [T], zeroed by the launcher
  float *grad;               // [T][k] or nullptr
  Layout L;
  ErrCtx e;
};

__device__ __forceinline__ float block_sum(float v, float *red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) s += red[w];
  return s;
}

__device__ __forceinline__ float block_max(float v, float *red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = -INFINITY;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) s = fmaxf(s, red[w]);
  return s;
}

__global__ void __launch_bounds__(kThreads, 1) indexer_kl_kernel(const KlParams p) {
  pdl_prologue();
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16 *sq = reinterpret_cast<__nv_bfloat16 *>(smem);            // [128][kQStride]
  __nv_bfloat16 *skv = sq + kH * kQStride;                                 // [32][576]
  __shared__ float red[kThreads / 32];
  __shared__ float s_p[kKeysPerCta];          // target p of each slot
  __shared__ long long s_row[kKeysPerCta];    // physical row of each slot, -1 = padding
  __shared__ int s_pos[kKeysPerCta];
  const int t = blockIdx.x, j0 = blockIdx.y * kKeysPerCta, tid = threadIdx.x;
  const RowPos rp = row_position(p.L, t);
  const bool row_ok = rp.len <= cache_capacity(p.L);

  // ---- this CTA's slots
  if (tid < kKeysPerCta) {
    long long r = -1;
    int s = -1;
    const int j = j0 + tid;
    if (j < p.k) {
      s = __ldg(p.idx + (long long)t * p.k + j);
      if (s >= 0 && s <= rp.pos && row_ok) {
        r = key_row(p.L, rp.b, s, p.e, 0x700);
      } else if (s != -1) {
        raise_error(p.e, DEV_BOUNDS, 0x701);
      }
    }
    s_row[tid] = r;
    s_pos[tid] = r >= 0 ? s : -1;
  }
  // ---- the row's log-sum-exp of the indexer scores over its selected set
  float mx = -INFINITY;
  for (int j = tid; j < p.k; j += kThreads) {
    const int s = row_ok ? __ldg(p.idx + (long long)t * p.k + j) : -1;
    if (s >= 0 && s <= rp.pos) mx = fmaxf(mx, __ldg(p.scores + (long long)t * p.ld + s));
  }
  mx = block_max(mx, red);
  float se = 0.f;
  for (int j = tid; j < p.k; j += kThreads) {
    const int s = row_ok ? __ldg(p.idx + (long long)t * p.k + j) : -1;
    if (s >= 0 && s <= rp.pos) se += __expf(__ldg(p.scores + (long long)t * p.ld + s) - mx);
  }
  se = block_sum(se, red);
  const float lse_i = se > 0.f ? mx + logf(se) : INFINITY;

  // ---- query row and the chunk's latent rows into shared memory
  {
    const uint32_t *qg = reinterpret_cast<const uint32_t *>(p.q + (long long)t * kH * kDk);
    uint32_t *qs = reinterpret_cast<uint32_t *>(sq);
    for (int i = tid; i < kH * (kDk / 2); i += kThreads) {
      const int h = i / (kDk / 2), d2 = i % (kDk / 2);
      qs[h * (kQStride / 2) + d2] = qg[i];
    }
    const char *kvb = reinterpret_cast<const char *>(p.kv);
    for (int i = tid; i < kKeysPerCta * (kDk * 2 / 16); i += kThreads) {
      const int key = i / (kDk * 2 / 16), c = i % (kDk * 2 / 16);
      const long long r = s_row[key];
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r >= 0) v = *reinterpret_cast<const uint4 *>(kvb + r * (kDk * 2) + c * 16);
      reinterpret_cast<uint4 *>(skv + key * kDk)[c] = v;
    }
  }
  __syncthreads();

  // ---- z for (head h, 16 keys of this half), then exp(z - lse_h)
  const int h = tid & (kH - 1), half = tid >> 7;
  float acc[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) acc[u] = 0.f;
  const __nv_bfloat162 *qh = reinterpret_cast<const __nv_bfloat162 *>(sq + h * kQStride);
  const __nv_bfloat162 *kk = reinterpret_cast<const __nv_bfloat162 *>(skv + half * 16 * kDk);
  for (int d2 = 0; d2 < kDk / 2; ++d2) {
    const float2 qv = __bfloat1622float2(qh[d2]);
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const float2 kv2 = __bfloat1622float2(kk[u * (kDk / 2) + d2]);
      acc[u] = fmaf(qv.x, kv2.x, fmaf(qv.y, kv2.y, acc[u]));
    }
  }
  const float lse_h = row_ok ? __ldg(p.lse + (long long)t * kH + h) : 0.f;
  // exp(z - lse_h), summed over the warp's 32 heads, then over the 4 warps of this half
  for (int u = 0; u < 16; ++u) {
    const bool live = s_row[half * 16 + u] >= 0;
    float e = live ? __expf(fmaf(acc[u], p.scale, -lse_h)) : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) e += __shfl_xor_sync(0xFFFFFFFFu, e, off);
    acc[u] = e;  // the warp's 32-head sum, in every lane
  }
  __shared__ float s_wsum[kThreads / 32][16];
  if ((tid & 31) == 0)
#pragma unroll
    for (int u = 0; u < 16; ++u) s_wsum[tid >> 5][u] = acc[u];
  __syncthreads();
  if (tid < kKeysPerCta) {
    const int hf = tid / 16, u = tid % 16;  // slot tid = half hf, key u of that half
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) s += s_wsum[hf * 4 + w][u];
    s_p[tid] = s / kH;
  }
  __syncthreads();

  // ---- loss terms and gradient per slot
  float c = 0.f;
  if (tid < kKeysPerCta) {
    const int j = j0 + tid;
    const float pj = s_p[tid];
    float g = 0.f;
    if (s_row[tid] >= 0) {
      const float lr = __ldg(p.scores + (long long)t * p.ld + s_pos[tid]) - lse_i;  // log r
      g = __expf(lr) - pj;
      if (pj > 0.f) c = pj * (logf(pj) - lr);
    }
    if (p.grad != nullptr && j < p.k) p.grad[(long long)t * p.k + j] = g;
  }
  c = block_sum(c, red);
  if (tid == 0 && row_ok) atomicAdd(p.loss + t, c);
}

}  // namespace

cudaError_t launch_indexer_kl(const void *q, const void *kv, int T, float scale, const int *idx, int k,
                              const float *lse, const float *scores, long long ld, const Layout &L, float *loss,
                              float *grad, const ErrCtx &e, cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(indexer_kl_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (err != cudaSuccess) return err;
  err = cudaMemsetAsync(loss, 0, sizeof(float) * (size_t)T, stream);
  if (err != cudaSuccess) return err;
  KlParams p;
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.kv = static_cast<const __nv_bfloat16 *>(kv);
  p.idx = idx;
  p.k = k;
  p.lse = lse;
  p.scores = scores;
  p.ld = ld;
  p.scale = scale;
  p.loss = loss;
  p.grad = grad;
  p.L = L;
  p.e = e;
  return launch_kernel(indexer_kl_kernel, dim3(T, (k + kKeysPerCta - 1) / kKeysPerCta), dim3(kThreads), kSmem, stream,
                       0, p);
}

}  // namespace dsa
