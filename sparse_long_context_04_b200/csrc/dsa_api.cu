// C ABI of the DSA hot path: host-side validation, kernel dispatch, chunking of
// long prefills, and the device error word. See include/dsa.h for the contract.
#include <mutex>
#include <stdio.h>
#include <string.h>

#include "dsa.h"
#include "internal.h"

namespace {

using dsa::ErrCtx;
using dsa::Layout;

// Device error word: [0] flags, [1] first failing site. One copy per device.
__device__ unsigned g_dsa_err[2];

unsigned long long g_wait_limit_ns = 1000000000ULL;
constexpr int kMaxDevices = 64;
unsigned *g_err_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};
std::mutex g_mu;

bool current_device(int *dev) { return cudaGetDevice(dev) == cudaSuccess && *dev >= 0 && *dev < kMaxDevices; }

// Per-device set-up on first use: address of the error word, SM count.
bool device_ctx(ErrCtx *e, int *sms) {
  int dev;
  if (!current_device(&dev)) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dsa_err) != cudaSuccess) return false;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    g_err_ptr[dev] = static_cast<unsigned *>(p);
    g_num_sms[dev] = n;
  }
  e->word = g_err_ptr[dev];
  e->limit = g_wait_limit_ns;
  *sms = g_num_sms[dev];
  return true;
}

bool a16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dsa_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return DSA_OK;
  cudaGetLastError();  // clear a sticky launch error so the next call starts clean
  return DSA_ERR_CUDA;
}

// Checks of the sequence layout common to every stage.
dsa_status check_layout(const dsa_seq_layout *lay, int T, Layout *L) {
  if (!lay || lay->batch < 1 || !lay->seq_lens || lay->n_max < 1 || T < 0) return DSA_ERR_INVALID_ARG;
  if (lay->page_size != 0 && lay->page_size != 64) return DSA_ERR_UNSUPPORTED;
  if (lay->page_size) {
    if (!lay->page_table || lay->max_pages < 1 || lay->num_pages < 1) return DSA_ERR_INVALID_ARG;
  }
  if (!lay->cu_q && T != lay->batch) return DSA_ERR_INVALID_ARG;
  L->row0 = 0;
  L->batch = lay->batch;
  L->seq_lens = lay->seq_lens;
  L->cu_q = lay->cu_q;
  L->page_size = lay->page_size;
  L->page_table = lay->page_table;
  L->max_pages = lay->max_pages;
  L->num_pages = lay->num_pages;
  L->n_max = lay->n_max;
  return DSA_OK;
}

long long capacity(const Layout &L) {
  return L.page_size ? (long long)L.max_pages * L.page_size : (long long)L.n_max;
}

// ---------------------------------------------------------------- stage checks
dsa_status check_indexer(const void *q_idx, const float *q_scale, const void *k_idx, const float *k_scale,
                         dsa_dtype dt, const float *w, int H_I, int d_I, const Layout &L, const float *scores,
                         long long ld) {
  if (!q_idx || !k_idx || !w || !scores || H_I < 1 || d_I < 1) return DSA_ERR_INVALID_ARG;
  if (ld < capacity(L) || (ld & 3)) return DSA_ERR_INVALID_ARG;
  if (dt == DSA_E4M3) {
    if (!q_scale) return DSA_ERR_INVALID_ARG;
    if (L.page_size == 0 && !k_scale) return DSA_ERR_INVALID_ARG;
    if (L.page_size != 0 && k_scale) return DSA_ERR_INVALID_ARG;
    if (H_I != 64 || d_I != 128) return DSA_ERR_UNSUPPORTED;
    if (!a16(q_idx) || !a16(k_idx) || !a16(scores) || !a16(w)) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
  }
  if (dt == DSA_F32) {
    if (q_scale || k_scale) return DSA_ERR_INVALID_ARG;
    if (L.page_size) return DSA_ERR_UNSUPPORTED;
    if ((long long)H_I * d_I > 8192) return DSA_ERR_UNSUPPORTED;
    return DSA_OK;
  }
  return DSA_ERR_UNSUPPORTED;
}

dsa_status run_indexer(const void *q_idx, const float *q_scale, const void *k_idx, const float *k_scale,
                       dsa_dtype dt, const float *w, int T, int H_I, int d_I, const Layout &L, float *scores,
                       long long ld, const ErrCtx &e, int sms, cudaStream_t st) {
  if (T == 0) return DSA_OK;
  if (dt == DSA_E4M3)
    return from_cuda(dsa::launch_indexer_fp8(static_cast<const uint8_t *>(q_idx), q_scale,
                                             static_cast<const uint8_t *>(k_idx), k_scale, w, T, L, scores, ld, e,
                                             sms, st));
  return from_cuda(dsa::launch_indexer_f32(static_cast<const float *>(q_idx), static_cast<const float *>(k_idx), w,
                                           T, H_I, d_I, L, scores, ld, e, st));
}

constexpr int kTopkCapMax = 32768;  // keys per CTA in shared memory (128 KiB)

dsa_status plan_topk(const Layout &L, int T, int sms, int *C_out, int *cap_out) {
  const long long capn = capacity(L);
  int C = 1;
  while ((long long)C * kTopkCapMax < capn) C *= 2;
  if (C > 8) return DSA_ERR_UNSUPPORTED;
  while (C < 8 && (long long)T * C * 2 <= sms && (capn + 2 * C - 1) / (2 * C) >= 2048) C *= 2;
  const long long per = (capn + C - 1) / C;
  *C_out = C;
  *cap_out = (int)((per + 31) / 32 * 32);
  return DSA_OK;
}

dsa_status run_topk(const float *scores, long long ld, int T, int k, const Layout &L, int *idx, const ErrCtx &e,
                    int sms, cudaStream_t st) {
  if (T == 0) return DSA_OK;
  int C, cap;
  dsa_status s = plan_topk(L, T, sms, &C, &cap);
  if (s != DSA_OK) return s;
  return from_cuda(dsa::launch_topk(scores, ld, T, k, L, C, cap, idx, e, st));
}

dsa_status check_attn(const void *q, const void *kv, dsa_dtype dt, int H, int Dk, int Dv, const int *idx, int k,
                      const Layout &L, const void *out) {
  if (!q || !kv || !idx || !out || H < 1 || Dk < 1 || Dv < 1 || Dv > Dk || k < 1) return DSA_ERR_INVALID_ARG;
  if (dt == DSA_BF16) {
    if (H != 128 || Dk != 576 || Dv != 512 || k > 16384) return DSA_ERR_UNSUPPORTED;
    if (!a16(q) || !a16(kv) || !a16(out)) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
  }
  if (dt == DSA_F32) {
    if (L.page_size) return DSA_ERR_UNSUPPORTED;
    if (H > 1024 || Dk > 1024 || Dv > 1024 || k > 8192) return DSA_ERR_UNSUPPORTED;
    return DSA_OK;
  }
  return DSA_ERR_UNSUPPORTED;
}

size_t attn_ws(int T, int k, dsa_dtype dt, int sms) {
  if (dt != DSA_BF16 || T <= 0) return 0;
  return dsa::attn_bf16_workspace(T, k, sms);
}

dsa_status run_attn(const void *q, const void *kv, dsa_dtype dt, int T, int H, int Dk, int Dv, float scale,
                    const int *idx, int k, const Layout &L, void *out, float *lse, void *ws, size_t ws_bytes,
                    const ErrCtx &e, int sms, cudaStream_t st) {
  if (T == 0) return DSA_OK;
  if (dt == DSA_BF16) {
    const size_t need = attn_ws(T, k, dt, sms);
    if (ws_bytes < need || (need && !ws) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return DSA_ERR_WORKSPACE;
    return from_cuda(dsa::launch_attn_bf16(q, kv, T, scale, idx, k, L, out, lse, ws, ws_bytes, e, sms, st));
  }
  return from_cuda(dsa::launch_attn_f32(static_cast<const float *>(q), static_cast<const float *>(kv), T, H, Dk, Dv,
                                        scale, idx, k, L, static_cast<float *>(out), lse, e, st));
}

// ---------------------------------------------------------------- forward plan
constexpr size_t kScoreChunkBytes = size_t(1) << 30;  // score rows per prefill chunk

constexpr long long kFusedMaxKeys = 262144;   // rows the candidate top-k's position bitmap covers

struct FwdPlan {
  long long ld;
  int rows_per_chunk;
  bool fused;  // decode + E4M3: indexer candidates and histograms, no score rows
  size_t off_scores, off_idx, off_attn, total;
  size_t off_hist, off_count, off_cscore, off_cpos;  // fused only
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool fwd_plan(const dsa_forward_args *a, int sms, FwdPlan *p) {
  if (!a || a->T < 0 || a->topk_path < DSA_TOPK_AUTO || a->topk_path > DSA_TOPK_FUSED) return false;
  const long long capn = a->lay.page_size ? (long long)a->lay.max_pages * a->lay.page_size : a->lay.n_max;
  if (capn < 1) return false;
  p->ld = (capn + 3) / 4 * 4;
  // the fused pair is exact on every decode shape it takes; it is not yet the faster
  // one on B200, so only an explicit request selects it
  p->fused = a->topk_path == DSA_TOPK_FUSED && a->lay.cu_q == nullptr && a->idx_dt == DSA_E4M3 &&
             capn <= kFusedMaxKeys;
  long long rows = (long long)(kScoreChunkBytes / (size_t)(p->ld * 4));
  if (rows < 1) rows = 1;
  if (rows > a->T) rows = a->T;
  if (a->lay.cu_q == nullptr) rows = a->T;  // decode: all rows at once
  p->rows_per_chunk = (int)(rows < 1 ? 1 : rows);
  size_t off = 0;
  p->off_scores = off;
  if (p->fused) {
    const size_t T = (size_t)a->T;
    p->off_hist = off;
    p->off_count = off + T * 4096 * 4;
    p->off_cscore = align256(p->off_count + T * 4);
    p->off_cpos = align256(p->off_cscore + T * (size_t)p->ld * 4);
    off = align256(p->off_cpos + T * (size_t)p->ld * 4);
  } else {
    off = align256(off + (size_t)p->rows_per_chunk * p->ld * 4);
  }
  p->off_idx = off;
  if (!a->idx_out) off = align256(off + (size_t)a->T * a->k * 4);
  p->off_attn = off;
  off = align256(off + attn_ws(a->T, a->k, a->attn_dt, sms));
  p->total = off;
  return true;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

int dsa_version(void) { return 100; }

const char *dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case DSA_ERR_CUDA: return "CUDA runtime error";
    case DSA_ERR_TIMEOUT: return "on-device wait timed out";
    case DSA_ERR_WORKSPACE: return "workspace missing or too small";
    case DSA_ERR_DEVICE_CHECK: return "device-side bounds check failed";
    case DSA_ERR_TOO_LARGE: return "call needs more scratch than the built-in scratch array holds";
  }
  return "unknown status";
}

dsa_status dsa_set_wait_limit_ns(unsigned long long ns) {
  if (ns == 0) return DSA_ERR_INVALID_ARG;
  g_wait_limit_ns = ns;
  return DSA_OK;
}

dsa_status dsa_get_device_error_site(void *stream, unsigned *site) {
  if (site) *site = 0;
  ErrCtx e;
  int sms;
  if (!device_ctx(&e, &sms)) return DSA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return from_cuda(cudaErrorUnknown);
  unsigned h[2] = {0, 0};
  if (cudaMemcpy(h, e.word, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  if (h[0] == 0) return DSA_OK;
  if (site) *site = h[1];
  const unsigned zero[2] = {0, 0};
  if (cudaMemcpy(e.word, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return DSA_ERR_CUDA;
  return (h[0] & dsa::DEV_TIMEOUT) ? DSA_ERR_TIMEOUT : DSA_ERR_DEVICE_CHECK;
}

dsa_status dsa_get_device_error(void *stream) { return dsa_get_device_error_site(stream, nullptr); }

dsa_status dsa_indexer_scores(const void *q_idx, const float *q_scale, const void *k_idx, const float *k_scale,
                              dsa_dtype dt, const float *w, int T, int H_I, int d_I, const dsa_seq_layout *lay,
                              float *scores, long long ld, void *stream) {
  Layout L;
  dsa_status s = check_layout(lay, T, &L);
  if (s != DSA_OK) return s;
  s = check_indexer(q_idx, q_scale, k_idx, k_scale, dt, w, H_I, d_I, L, scores, ld);
  if (s != DSA_OK) return s;
  ErrCtx e;
  int sms;
  if (!device_ctx(&e, &sms)) return DSA_ERR_CUDA;
  return run_indexer(q_idx, q_scale, k_idx, k_scale, dt, w, T, H_I, d_I, L, scores, ld, e, sms,
                     static_cast<cudaStream_t>(stream));
}

dsa_status dsa_topk(const float *scores, long long ld, int T, int k, const dsa_seq_layout *lay, int *idx,
                    void *stream) {
  Layout L;
  dsa_status s = check_layout(lay, T, &L);
  if (s != DSA_OK) return s;
  if (!scores || !idx || k < 1 || !a16(scores) || (ld & 3) || ld < capacity(L)) return DSA_ERR_INVALID_ARG;
  ErrCtx e;
  int sms;
  if (!device_ctx(&e, &sms)) return DSA_ERR_CUDA;
  return run_topk(scores, ld, T, k, L, idx, e, sms, static_cast<cudaStream_t>(stream));
}

size_t dsa_sparse_mqa_attn_workspace_size(int T, int H, int Dv, int k, dsa_dtype dt) {
  (void)H;
  (void)Dv;
  ErrCtx e;
  int sms;
  if (!device_ctx(&e, &sms)) return 0;
  return attn_ws(T, k, dt, sms);
}

dsa_status dsa_topk_from_candidates(const float *score, const int *pos, const int *count, long long cap,
                                    const unsigned *hist, int T, int k, const dsa_seq_layout *lay, int *idx,
                                    void *stream) {
  Layout L;
  dsa_status s = check_layout(lay, T, &L);
  if (s != DSA_OK) return s;
  if (!score || !pos || !count || !hist || !idx || k < 1 || cap < 1) return DSA_ERR_INVALID_ARG;
  if (capacity(L) > 262144) return DSA_ERR_UNSUPPORTED;
  if (T == 0) return DSA_OK;
  ErrCtx e;
  int sms;
  if (!device_ctx(&e, &sms)) return DSA_ERR_CUDA;
  return from_cuda(dsa::launch_topk_candidates(score, pos, count, cap, hist, T, k, L, idx, e,
                                               static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_indexer_candidates(const void *q_idx, const float *q_scale, const void *k_idx, const float *k_scale,
                                  dsa_dtype dt, const float *w, int T, int H_I, int d_I, const dsa_seq_layout *lay,
                                  int k, unsigned *hist, float *cand_score, int *cand_pos, int *cand_count,
                                  long long cap, void *stream) {
  Layout L;
  dsa_status s = check_layout(lay, T, &L);
  if (s != DSA_OK) return s;
  if (L.cu_q != nullptr || dt != DSA_E4M3) return DSA_ERR_UNSUPPORTED;
  // the score buffer check is skipped (no scores are written): pass a dummy that passes it
  s = check_indexer(q_idx, q_scale, k_idx, k_scale, dt, w, H_I, d_I, L, reinterpret_cast<const float *>(16),
                    (capacity(L) + 3) / 4 * 4);
  if (s != DSA_OK) return s;
  if (!hist || !cand_score || !cand_pos || !cand_count || k < 1) return DSA_ERR_INVALID_ARG;
  if (cap < capacity(L)) return DSA_ERR_INVALID_ARG;
  const uintptr_t a4 = reinterpret_cast<uintptr_t>(cand_score) | reinterpret_cast<uintptr_t>(cand_pos) |
                       reinterpret_cast<uintptr_t>(cand_count);
  if ((a4 & 3u) || !a16(hist)) return DSA_ERR_INVALID_ARG;
  if (T == 0) return DSA_OK;
  ErrCtx e;
  int sms;
  if (!device_ctx(&e, &sms)) return DSA_ERR_CUDA;
  return from_cuda(dsa::launch_indexer_fp8_fused(static_cast<const uint8_t *>(q_idx), q_scale,
                                                 static_cast<const uint8_t *>(k_idx), k_scale, w, T, L, k, hist,
                                                 cand_count, cand_score, cand_pos, cap, e, sms,
                                                 static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_sparse_mqa_attn(const void *q, const void *kv, dsa_dtype dt, int T, int H, int Dk, int Dv,
                               float softmax_scale, const int *idx, int k, const dsa_seq_layout *lay, void *out,
                               float *lse, void *workspace, size_t ws_bytes, void *stream) {
  Layout L;
  dsa_status s = check_layout(lay, T, &L);
  if (s != DSA_OK) return s;
  s = check_attn(q, kv, dt, H, Dk, Dv, idx, k, L, out);
  if (s != DSA_OK) return s;
  ErrCtx e;
  int sms;
  if (!device_ctx(&e, &sms)) return DSA_ERR_CUDA;
  return run_attn(q, kv, dt, T, H, Dk, Dv, softmax_scale, idx, k, L, out, lse, workspace, ws_bytes, e, sms,
                  static_cast<cudaStream_t>(stream));
}

dsa_status dsa_sparse_mqa_attn_noalloc(const void *q, const void *kv, dsa_dtype dt, int T, int H, int Dk, int Dv,
                                       float softmax_scale, const int *idx, int k, const dsa_seq_layout *lay,
                                       void *out, float *lse, void *stream) {
  Layout L;
  dsa_status s = check_layout(lay, T, &L);
  if (s != DSA_OK) return s;
  s = check_attn(q, kv, dt, H, Dk, Dv, idx, k, L, out);
  if (s != DSA_OK) return s;
  if (dt != DSA_BF16) return DSA_ERR_UNSUPPORTED;
  if (dsa::attn_bf16_scratch_bytes(T, k) > dsa::attn_bf16_scratch_limit()) return DSA_ERR_TOO_LARGE;
  ErrCtx e;
  int sms;
  if (!device_ctx(&e, &sms)) return DSA_ERR_CUDA;
  if (T == 0) return from_cuda(dsa::attn_bf16_scratch_setup());  // set-up only: a cheap first call
  return from_cuda(dsa::launch_attn_bf16_noalloc(q, kv, T, softmax_scale, idx, k, L, out, lse, e, sms,
                                                 static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_cache_append(const void *k_new, dsa_dtype k_dt, const void *kv_new, int T, int d_I, int Dk,
                            const dsa_seq_layout *lay, void *k_cache, float *k_scale, void *kv_cache, void *stream) {
  Layout L;
  dsa_status s = check_layout(lay, T, &L);
  if (s != DSA_OK) return s;
  if (!k_new || !k_cache) return DSA_ERR_INVALID_ARG;
  if (k_dt != DSA_F32 && k_dt != DSA_BF16) return DSA_ERR_UNSUPPORTED;
  if (d_I != 128) return DSA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(k_new) & (k_dt == DSA_F32 ? 15u : 7u)) != 0) return DSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k_cache) & 3u) != 0) return DSA_ERR_INVALID_ARG;
  if (L.page_size ? k_scale != nullptr : (k_scale == nullptr || (reinterpret_cast<uintptr_t>(k_scale) & 3u)))
    return DSA_ERR_INVALID_ARG;
  if (kv_new) {
    if (!kv_cache || Dk < 8 || Dk > 4096 || (Dk % 8) != 0 || !a16(kv_new) || !a16(kv_cache))
      return DSA_ERR_INVALID_ARG;
  }
  if (T == 0) return DSA_OK;
  ErrCtx e;
  int sms;
  if (!device_ctx(&e, &sms)) return DSA_ERR_CUDA;
  return from_cuda(dsa::launch_cache_append(k_new, k_dt == DSA_BF16, kv_new, T, Dk, L, k_cache, k_scale, kv_cache, e,
                                            static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_indexer_kl(const void *q, const void *kv, dsa_dtype dt, int T, int H, int Dk, float softmax_scale,
                          const int *idx, int k, const dsa_seq_layout *lay, const float *lse, const float *scores,
                          long long ld, float *loss, float *grad, void *stream) {
  Layout L;
  dsa_status s = check_layout(lay, T, &L);
  if (s != DSA_OK) return s;
  if (!q || !kv || !idx || !lse || !scores || !loss || k < 1 || H < 1 || Dk < 1) return DSA_ERR_INVALID_ARG;
  const long long capn = L.page_size ? (long long)L.max_pages * L.page_size : L.n_max;
  if (ld < capn) return DSA_ERR_INVALID_ARG;
  if (dt != DSA_BF16 || H != 128 || Dk != 576 || k > 16384) return DSA_ERR_UNSUPPORTED;
  const uintptr_t a4 = reinterpret_cast<uintptr_t>(lse) | reinterpret_cast<uintptr_t>(scores) |
                       reinterpret_cast<uintptr_t>(loss) | reinterpret_cast<uintptr_t>(grad) |
                       reinterpret_cast<uintptr_t>(idx);
  if ((a4 & 3u) != 0 || !a16(q) || !a16(kv)) return DSA_ERR_INVALID_ARG;  // q is read by TMA
  if (T == 0) return DSA_OK;
  ErrCtx e;
  int sms;
  if (!device_ctx(&e, &sms)) return DSA_ERR_CUDA;
  return from_cuda(dsa::launch_indexer_kl(q, kv, T, softmax_scale, idx, k, lse, scores, ld, L, loss, grad, e, sms,
                                          static_cast<cudaStream_t>(stream)));
}

size_t dsa_sparse_mqa_attn_backward_workspace_size(int T) { return T > 0 ? dsa::attn_bwd_workspace(T) : 0; }

dsa_status dsa_sparse_mqa_attn_backward(const void *q, const void *kv, dsa_dtype dt, int T, int H, int Dk, int Dv,
                                        float softmax_scale, const int *idx, int k, const dsa_seq_layout *lay,
                                        const void *out, const void *dout, const float *lse, float *dq, float *dkv,
                                        void *workspace, size_t ws_bytes, void *stream) {
  Layout L;
  dsa_status s = check_layout(lay, T, &L);
  if (s != DSA_OK) return s;
  if (!q || !kv || !idx || !out || !dout || !lse || !dq || !dkv || k < 1 || H < 1 || Dk < 1 || Dv < 1 || Dv > Dk)
    return DSA_ERR_INVALID_ARG;
  if (dt != DSA_BF16 || H != 128 || Dk != 576 || Dv != 512 || k > 16384) return DSA_ERR_UNSUPPORTED;
  if (!a16(q) || !a16(kv) || !a16(out) || !a16(dout) || !a16(dq) || !a16(dkv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) != 0 || (reinterpret_cast<uintptr_t>(idx) & 3u) != 0)
    return DSA_ERR_INVALID_ARG;
  if (T == 0) return DSA_OK;
  if (ws_bytes < dsa::attn_bwd_workspace(T) || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return DSA_ERR_WORKSPACE;
  ErrCtx e;
  int sms;
  if (!device_ctx(&e, &sms)) return DSA_ERR_CUDA;
  return from_cuda(dsa::launch_attn_bwd(q, kv, T, softmax_scale, idx, k, L, out, dout, lse, dq, dkv, workspace, e,
                                        static_cast<cudaStream_t>(stream)));
}

size_t dsa_forward_workspace_size(const dsa_forward_args *a) {
  ErrCtx e;
  int sms;
  if (!device_ctx(&e, &sms)) return 0;
  FwdPlan p;
  if (!fwd_plan(a, sms, &p)) return 0;
  return p.total;
}

dsa_status dsa_forward(const dsa_forward_args *a, void *workspace, size_t ws_bytes, void *stream) {
  if (!a) return DSA_ERR_INVALID_ARG;
  Layout L;
  dsa_status s = check_layout(&a->lay, a->T, &L);
  if (s != DSA_OK) return s;
  ErrCtx e;
  int sms;
  if (!device_ctx(&e, &sms)) return DSA_ERR_CUDA;
  FwdPlan p;
  if (!fwd_plan(a, sms, &p)) return DSA_ERR_INVALID_ARG;
  s = check_indexer(a->q_idx, a->q_scale, a->k_idx, a->k_scale, a->idx_dt, a->w, a->H_I, a->d_I, L,
                    reinterpret_cast<const float *>(16), p.ld);
  if (s != DSA_OK) return s;
  s = check_attn(a->q, a->kv, a->attn_dt, a->H, a->Dk, a->Dv, reinterpret_cast<const int *>(16), a->k, L, a->out);
  if (s != DSA_OK) return s;
  if (a->T == 0) return DSA_OK;
  if (ws_bytes < p.total || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  float *scores = reinterpret_cast<float *>(ws + p.off_scores);
  int *idx = a->idx_out ? a->idx_out : reinterpret_cast<int *>(ws + p.off_idx);

  if (p.fused) {
    unsigned *hist = reinterpret_cast<unsigned *>(ws + p.off_hist);
    int *count = reinterpret_cast<int *>(ws + p.off_count);
    float *cscore = reinterpret_cast<float *>(ws + p.off_cscore);
    int *cpos = reinterpret_cast<int *>(ws + p.off_cpos);
    s = from_cuda(dsa::launch_indexer_fp8_fused(static_cast<const uint8_t *>(a->q_idx), a->q_scale,
                                                static_cast<const uint8_t *>(a->k_idx), a->k_scale, a->w, a->T, L,
                                                a->k, hist, count, cscore, cpos, p.ld, e, sms, st));
    if (s != DSA_OK) return s;
    s = from_cuda(dsa::launch_topk_candidates(cscore, cpos, count, p.ld, hist, a->T, a->k, L, idx, e, st));
    if (s != DSA_OK) return s;
    return run_attn(a->q, a->kv, a->attn_dt, a->T, a->H, a->Dk, a->Dv, a->softmax_scale, idx, a->k, L, a->out,
                    a->lse, ws + p.off_attn, p.total - p.off_attn, e, sms, st);
  }
  const size_t qrow = (size_t)a->H_I * a->d_I * (a->idx_dt == DSA_E4M3 ? 1 : 4);
  for (int r0 = 0; r0 < a->T; r0 += p.rows_per_chunk) {
    const int n = (a->T - r0 < p.rows_per_chunk) ? a->T - r0 : p.rows_per_chunk;
    Layout Lc = L;
    Lc.row0 = r0;
    s = run_indexer(static_cast<const char *>(a->q_idx) + (size_t)r0 * qrow, a->q_scale ? a->q_scale + r0 : nullptr,
                    a->k_idx, a->k_scale, a->idx_dt, a->w + (size_t)r0 * a->H_I, n, a->H_I, a->d_I, Lc, scores,
                    p.ld, e, sms, st);
    if (s != DSA_OK) return s;
    s = run_topk(scores, p.ld, n, a->k, Lc, idx + (size_t)r0 * a->k, e, sms, st);
    if (s != DSA_OK) return s;
  }
  return run_attn(a->q, a->kv, a->attn_dt, a->T, a->H, a->Dk, a->Dv, a->softmax_scale, idx, a->k, L, a->out,
                  a->lse, ws + p.off_attn, p.total - p.off_attn, e, sms, st);
}

}  // extern "C"
