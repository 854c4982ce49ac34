// Cache write of the decode loop: each query row's new indexer key, quantised to
// FP8 e4m3 with one fp32 scale per token, and its latent KV row go into the row's
// own position of the caches the other stages read.
//
// mundobytes.com "Deepseek-v3-2-exp": served with 64-token KV pages (the launch
// line of the deployment section) and with the indexer kernels published in a
// paged version (open-kernels paragraph); jdon.com "DeepSeek-V3.2-Exp": the
// indexer runs in FP8. Per-token quantisation: scale = max|x| / 448 (1 for an
// all-zero row), code = e4m3 value nearest to x / scale, ties to even,
// saturating; the paged indexer cache holds [64 x 128 code bytes][64 fp32
// scales] per page (8448 bytes), the latent cache [64][Dk] bf16 per page.
//
// One CTA per row: warp 0 quantises the 128-value key (4 values per lane, a warp
// max for the scale), the other three warps copy the latent row in 16-byte pieces.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int kDI = 128;
constexpr int kThreads = 128;
constexpr int kPageKeyBytes = 64 * kDI;        // code bytes of a page
constexpr int kPageBytes = kPageKeyBytes + 64 * 4;  // + scales

struct AppendParams {
  const void *k_new;             // [T][128] fp32 or bf16
  int k_bf16;
  const __nv_bfloat16 *kv_new;   // [T][Dk] or nullptr
  int Dk;
  uint8_t *k_cache;              // paged: [pages][8448]; contiguous: [B][n_max][128]
  float *k_scale;                // contiguous only: [B][n_max]
  __nv_bfloat16 *kv_cache;       // paged: [pages*64][Dk]; contiguous: [B][n_max][Dk]
  Layout L;
  ErrCtx e;
};

__global__ void __launch_bounds__(kThreads) cache_append_kernel(const AppendParams p) {
  pdl_prologue();
  const int t = blockIdx.x;
  const RowPos rp = row_position(p.L, t);
  if (rp.pos < 0 || rp.len > cache_capacity(p.L)) {
    if (threadIdx.x == 0) raise_error(p.e, DEV_BOUNDS, 0x600);
    return;
  }
  const long long row = key_row(p.L, rp.b, rp.pos, p.e, 0x601);
  if (row < 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    float x[4];
    if (p.k_bf16) {
      const uint2 raw = *reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(p.k_new) +
                                                         (long long)t * kDI + lane * 4);
      const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
      const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
      x[0] = a.x;
      x[1] = a.y;
      x[2] = b.x;
      x[3] = b.y;
    } else {
      const float4 v = *reinterpret_cast<const float4 *>(static_cast<const float *>(p.k_new) +
                                                         (long long)t * kDI + lane * 4);
      x[0] = v.x;
      x[1] = v.y;
      x[2] = v.z;
      x[3] = v.w;
    }
    float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    const float scale = amax > 0.f ? amax / 448.f : 1.f;
    uint32_t packed = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // IEEE division, then the saturating round-to-nearest-even conversion
      const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(x[j] / scale, __NV_SATFINITE, __NV_E4M3);
      packed |= (uint32_t)c << (8 * j);
    }
    if (p.L.page_size) {
      uint8_t *page = p.k_cache + (row / p.L.page_size) * (long long)kPageBytes;
      const int slot = (int)(row % p.L.page_size);
      *reinterpret_cast<uint32_t *>(page + slot * kDI + lane * 4) = packed;
      if (lane == 0) *reinterpret_cast<float *>(page + kPageKeyBytes + slot * 4) = scale;
    } else {
      *reinterpret_cast<uint32_t *>(p.k_cache + row * kDI + lane * 4) = packed;
      if (lane == 0) p.k_scale[row] = scale;
    }
  } else if (p.kv_new != nullptr) {
    const int pieces = p.Dk * 2 / 16;
    const uint4 *src = reinterpret_cast<const uint4 *>(p.kv_new + (long long)t * p.Dk);
    uint4 *dst = reinterpret_cast<uint4 *>(p.kv_cache + row * p.Dk);
    for (int c = threadIdx.x - 32; c < pieces; c += kThreads - 32) dst[c] = src[c];
  }
}

}  // namespace

cudaError_t launch_cache_append(const void *k_new, bool k_bf16, const void *kv_new, int T, int Dk, const Layout &L,
                                void *k_cache, float *k_scale, void *kv_cache, const ErrCtx &e, cudaStream_t stream) {
  AppendParams p;
  p.k_new = k_new;
  p.k_bf16 = k_bf16 ? 1 : 0;
  p.kv_new = static_cast<const __nv_bfloat16 *>(kv_new);
  p.Dk = Dk;
  p.k_cache = static_cast<uint8_t *>(k_cache);
  p.k_scale = k_scale;
  p.kv_cache = static_cast<__nv_bfloat16 *>(kv_cache);
  p.L = L;
  p.e = e;
  return launch_kernel(cache_append_kernel, dim3(T), dim3(kThreads), 0, stream, 0, p);
}

}  // namespace dsa
