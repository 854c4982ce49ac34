// Launchers behind the C ABI (host side). Each returns the CUDA error of its
// launch; argument validation happens in dsa_api.cu before any of them runs.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "common.cuh"

#include <utility>

namespace dsa {

// Launch with programmatic stream serialization (the kernel starts with
// pdl_prologue()) and, when cluster_x > 0, thread-block clusters of cluster_x CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          unsigned cluster_x, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// top-k (topk.cu): C CTAs per row (cluster), `cap` keys of shared memory per CTA
size_t topk_smem_bytes(int cap);
cudaError_t launch_topk(const float *scores, long long ld, int T, int k, const Layout &L, int C, int cap, int *idx,
                        const ErrCtx &e, cudaStream_t stream);

// plain fp32 kernels on CUDA cores (fp32_path.cu)
cudaError_t launch_indexer_f32(const float *q, const float *kI, const float *w, int T, int H_I, int d_I,
                               const Layout &L, float *scores, long long ld, const ErrCtx &e, cudaStream_t stream);
cudaError_t launch_attn_f32(const float *q, const float *kv, int T, int H, int Dk, int Dv, float scale,
                            const int *idx, int k, const Layout &L, float *out, float *lse, const ErrCtx &e,
                            cudaStream_t stream);

// FP8 tcgen05 lightning indexer (indexer_fp8.cu): H_I = 64, d_I = 128
int indexer_fp8_grid(int num_sms);
cudaError_t launch_indexer_fp8(const uint8_t *q, const float *q_scale, const uint8_t *kI, const float *k_scale,
                               const float *w, int T, const Layout &L, float *scores, long long ld, const ErrCtx &e,
                               int num_sms, cudaStream_t stream);

// the same indexer for decode rows with the producer half of the fused top-k: instead
// of the scores, the keys at or above a refreshed lower bound of each row's threshold
// bin and their 12-bit order-key histogram (hist and cand_count are cleared first, by a
// kernel on the same stream)
cudaError_t launch_indexer_fp8_fused(const uint8_t *q, const float *q_scale, const uint8_t *kI, const float *k_scale,
                                     const float *w, int T, const Layout &L, int k, unsigned *hist, int *cand_count,
                                     float *cand_score, int *cand_pos, long long cand_cap, const ErrCtx &e,
                                     int num_sms, cudaStream_t stream);

// bf16 tcgen05 sparse MQA attention (attn_bf16.cu): H = 128, Dk = 576, Dv = 512
struct AttnPlan {
  int keys_per_split;  // multiple of 64, <= 256
  int splits;          // per query row
};
AttnPlan attn_bf16_plan(int T, int k, int num_sms);
size_t attn_bf16_workspace(int T, int k, int num_sms);
cudaError_t launch_attn_bf16(const void *q, const void *kv, int T, float scale, const int *idx, int k,
                             const Layout &L, void *out, float *lse, void *ws, size_t ws_bytes, const ErrCtx &e,
                             int num_sms, cudaStream_t stream);

// same attention with its partials in the library's static scratch array
size_t attn_bf16_scratch_bytes(int T, int k);
size_t attn_bf16_scratch_limit();
// looks up the scratch array's address on the current device (first use per device)
cudaError_t attn_bf16_scratch_setup();
cudaError_t launch_attn_bf16_noalloc(const void *q, const void *kv, int T, float scale, const int *idx, int k,
                                     const Layout &L, void *out, float *lse, const ErrCtx &e, int num_sms,
                                     cudaStream_t stream);

// cache write (cache_append.cu): new indexer key (e4m3 + per-token scale) and latent row per query row
cudaError_t launch_cache_append(const void *k_new, bool k_bf16, const void *kv_new, int T, int Dk, const Layout &L,
                                void *k_cache, float *k_scale, void *kv_cache, const ErrCtx &e, cudaStream_t stream);

// TMA map of bf16 query rows of 576 values viewed as [rows][576]: boxes of 64 values x
// 128 rows (one head block), 128-byte swizzle (attn_bf16.cu)
bool make_q576_map(CUtensorMap *m, const void *q, unsigned long long rows);
// the same for bf16 rows of `width` values (a multiple of 64, rows 16-byte aligned)
bool make_bf16_rows_map(CUtensorMap *m, const void *base, unsigned long long rows, unsigned width);

// sparse attention backward (attn_bwd.cu): bf16, H = 128, Dk = 576, Dv = 512;
// the workspace holds dO . o per (row, head)
size_t attn_bwd_workspace(int T);
cudaError_t launch_attn_bwd(const void *q, const void *kv, int T, float scale, const int *idx, int k,
                            const Layout &L, const void *out, const void *dout, const float *lse, float *dq,
                            float *dkv, void *ws, const ErrCtx &e, cudaStream_t stream);

// top-k from a filtered candidate list and the rows' complete 12-bit histograms
// (topk_candidates.cu)
size_t topk_candidates_smem();
cudaError_t launch_topk_candidates(const float *score, const int *pos, const int *count, long long cap,
                                   const unsigned *hist, int T, int k, const Layout &L, int *idx, const ErrCtx &e,
                                   cudaStream_t stream);

// indexer loss on the selected set and its gradient (indexer_kl.cu): bf16, H = 128, Dk = 576
cudaError_t launch_indexer_kl(const void *q, const void *kv, int T, float scale, const int *idx, int k,
                              const float *lse, const float *scores, long long ld, const Layout &L, float *loss,
                              float *grad, const ErrCtx &e, int num_sms, cudaStream_t stream);

}  // namespace dsa
