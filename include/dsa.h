/*
 * dsa.h — C ABI of the DeepSeek Sparse Attention (DSA) hot path on B200 (sm_100a).
 *
 * The path has three stages, as the DeepSeek-V3.2-Exp pages describe them:
 *   1. lightning indexer  I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]),  s <= pos_t
 *        jdon.com "DeepSeek-V3.2-Exp", lightning-indexer paragraph (FP8, few heads,
 *        weighted sum of ReLU-activated dot products) and the "matchmaking" analogy
 *        paragraph (ReLU, w_I as weight, q_I and k_I scored on meeting);
 *        openi.cn "DeepSeek-V3.2", technical section, lightning-indexer item.
 *   2. fine-grained token selection: the k best-scoring earlier tokens per query
 *        jdon.com, sparse-training paragraph (K = 2048) and selection paragraph;
 *        openi.cn, token-selection item.
 *   3. sparse MQA attention over the selected latent rows (all heads share one row)
 *        jdon.com, selection paragraph (only the k chosen entries take part, output u_t);
 *        openi.cn, "MLA in MQA mode" item (one value entry shared by many queries).
 *
 * Conventions (every entry point):
 *   - Pointers marked "device" are CUDA device pointers owned by the caller; the
 *     library never allocates device memory and never frees caller memory.
 *   - `stream` is a cudaStream_t passed as void*; all work is enqueued
 *     asynchronously on it. NULL means the legacy default stream.
 *   - Argument errors are found on the host before any launch and return
 *     DSA_ERR_INVALID_ARG; valid shapes without a kernel return DSA_ERR_UNSUPPORTED.
 *     Nothing is launched when an error is returned.
 *   - Kernels check what only the device can see (sequence lengths against the
 *     cache extent, page ids against the pool, indices against the causal range):
 *     a violating access is skipped and recorded in a device error word, read
 *     back with dsa_get_device_error(). Every on-device wait is bounded; a wait
 *     that runs out records DSA_ERR_TIMEOUT there instead of hanging.
 *   - No C++ exception crosses this boundary.
 *
 * Query rows and positions. A call covers T query rows. With cu_q == NULL
 * (decode) row t is the newest token of sequence t: T == batch, pos_t =
 * seq_lens[t] - 1. With cu_q != NULL (prefill) rows cu_q[b] .. cu_q[b+1]-1 belong
 * to sequence b and are its last (cu_q[b+1]-cu_q[b]) tokens: the i-th of them sits
 * at pos = seq_lens[b] - (cu_q[b+1]-cu_q[b]) + i. The causal set of a row is
 * s = 0 .. pos_t, the row's own position included.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,   /* bad pointer, size, stride or alignment */
  DSA_ERR_UNSUPPORTED = 2,   /* valid arguments, no kernel for this shape/dtype */
  DSA_ERR_CUDA = 3,          /* a CUDA runtime call failed (launch, attribute) */
  DSA_ERR_TIMEOUT = 4,       /* an on-device wait ran out (device error word) */
  DSA_ERR_WORKSPACE = 5,     /* workspace missing or smaller than required */
  DSA_ERR_DEVICE_CHECK = 6,  /* a device-side bounds check failed (device error word) */
  DSA_ERR_TOO_LARGE = 7      /* the call needs more scratch than the library's built-in array */
} dsa_status;

typedef enum { DSA_F32 = 0, DSA_BF16 = 1, DSA_E4M3 = 2 } dsa_dtype;

/* Addressing of the key caches, shared by all stages. */
typedef struct {
  int batch;              /* B >= 1 sequences */
  const int *seq_lens;    /* device int32 [B]: keys held by each sequence (>= 1) */
  const int *cu_q;        /* device int32 [B+1] query-row offsets (prefill); NULL = decode */
  int page_size;          /* 0 = contiguous caches; 64 = paged caches */
  const int *page_table;  /* device int32 [B][max_pages] physical page ids (paged only) */
  int max_pages;          /* row length of page_table (paged only) */
  int num_pages;          /* pages in each cache pool (paged only; ids must be < num_pages) */
  int n_max;              /* host upper bound of seq_lens; contiguous caches are
                             laid out [B][n_max][...] */
} dsa_seq_layout;

/*
 * Stage 1 — lightning indexer scores.
 *   scores[t*ld + s] = sum_j w[t*H_I + j] * max(0, q~[t,j,:] . k~[s,:])  for s <= pos_t,
 * with q~ = q_scale[t] * dec(q_idx) and k~ = k_scale[s] * dec(k_idx) for E4M3
 * (per-token fp32 scales, > 0), or the plain values for F32.
 *   q_idx    device [T][H_I][d_I], E4M3 bytes or float32 (dt)
 *   q_scale  device float32 [T] (E4M3) or NULL (F32)
 *   k_idx    contiguous: device [B][n_max][d_I] (E4M3 bytes or float32);
 *            paged (E4M3 only): pool of num_pages pages, each page_size*d_I key
 *            bytes followed by page_size float32 scales (little-endian)
 *   k_scale  contiguous E4M3: device float32 [B][n_max]; otherwise NULL
 *   w        device float32 [T][H_I]
 *   scores   device float32 [T][ld], ld >= n_max and a multiple of 4; entries with
 *            s > pos_t are unspecified on return
 * Fast path: E4M3 with H_I = 64, d_I = 128 (tcgen05 FP8 MMA). F32: H_I*d_I <= 8192,
 * contiguous only. Buffers of the fast path must be 16-byte aligned.
 */
dsa_status dsa_indexer_scores(const void *q_idx, const float *q_scale,
                              const void *k_idx, const float *k_scale, dsa_dtype dt,
                              const float *w, int T, int H_I, int d_I,
                              const dsa_seq_layout *lay, float *scores, long long ld,
                              void *stream);

/*
 * Stage 2 — fine-grained top-k selection.
 * For each row t reads scores[t*ld + s], s = 0..pos_t, and writes idx[t*k + i]:
 * the m = min(k, pos_t+1) positions that come first under (score descending,
 * position ascending), in ascending position order, then k-m entries of -1.
 * -0.0 equals +0.0; NaN ranks below every number. Bit-exact, deterministic.
 *   scores  device float32 [T][ld], 16-byte aligned, ld a multiple of 4
 *   idx     device int32 [T][k]
 * Rows up to 262144 keys; k >= 1.
 */
dsa_status dsa_topk(const float *scores, long long ld, int T, int k,
                    const dsa_seq_layout *lay, int *idx, void *stream);

/*
 * Stage 2 from a filtered candidate list: the finishing half of an indexer ->
 * top-k that does not write its full score rows. Same result, order and tie rule
 * as dsa_topk over the row's complete scores.
 * Order key of a score x (the rule dsa_topk ranks by): 0 for NaN; otherwise, with
 * u the bits of x and -0 taken as +0, u | 0x80000000 for x >= 0 and ~u for x < 0.
 * The bin of x is its order key >> 20 (4096 bins).
 *   score, pos  device float32 / int32 [T][cap]: each row's candidates, any order,
 *           each position at most once. Every position whose bin is at or above
 *           the row's threshold bin (the bin of its k-th best key) must be there;
 *           a producer gets this by keeping each key whose bin is at or above any
 *           lower bound of the threshold bin, e.g. one read from a histogram of
 *           the row's keys so far (the highest bin with at least k keys at or above).
 *           Candidates below the threshold bin are ignored.
 *   hist    device uint32 [T][4096]: per row and bin, a count that is exact for
 *           every bin at or above the row's threshold bin (there it counts the
 *           row's scores in the bin, all of which are candidates), with at least
 *           min(k, pos_t + 1) in total; lower bins may hold any count. The
 *           histogram of all the row's scores qualifies, and so does the
 *           histogram of its candidates.
 *   count   device int32 [T]: candidates per row (<= cap)
 *   idx     device int32 [T][k], as dsa_topk writes it
 * Rows up to 262144 keys; k >= 1. A histogram or candidate list that breaks the
 * rules above (counts that disagree, a position out of range) is a device check
 * failure and the row is written as -1.
 */
dsa_status dsa_topk_from_candidates(const float *score, const int *pos, const int *count,
                                    long long cap, const unsigned *hist, int T, int k,
                                    const dsa_seq_layout *lay, int *idx, void *stream);

/*
 * Stages 1 and 2 fused, producer half (decode rows): the lightning indexer of
 * dsa_indexer_scores without writing the score rows. For each row it writes a
 * candidate list, which holds every key at or above a lower bound of the row's
 * threshold bin that is refreshed from the list's own histogram while the row is
 * scored, and that histogram (the candidates' order-key bins, as
 * dsa_topk_from_candidates reads them). dsa_topk_from_candidates on its outputs
 * gives exactly dsa_topk's selection over the scores dsa_indexer_scores would
 * write; the candidates' scores are those scores, bit for bit.
 * jdon.com "DeepSeek-V3.2-Exp": lightning-indexer paragraph (scores) and
 * sparse-training paragraph (K = 2048 kept per query).
 *   q_idx, q_scale, k_idx, k_scale, dt, w, H_I, d_I, lay: as for dsa_indexer_scores,
 *            decode layouts only (lay->cu_q == NULL, T == batch), E4M3, H_I = 64, d_I = 128
 *   k        the selection size the bound is kept for (>= 1)
 *   hist     device uint32 [T][4096], 16-byte aligned: per row, the candidates in each bin
 *   cand_count  device int32 [T]: candidates per row. hist and cand_count are
 *            cleared and written by the call.
 *   cand_score, cand_pos  device float32 / int32 [T][cap], cap >= the layout's cache
 *            capacity (max_pages * page_size, or n_max), so no row can overflow; the
 *            first cand_count[t] entries of row t are its candidates, in no order
 * cand_score, cand_pos, cand_count 4-byte aligned; q_idx, k_idx and w 16-byte aligned.
 */
dsa_status dsa_indexer_candidates(const void *q_idx, const float *q_scale,
                                  const void *k_idx, const float *k_scale, dsa_dtype dt,
                                  const float *w, int T, int H_I, int d_I,
                                  const dsa_seq_layout *lay, int k, unsigned *hist,
                                  float *cand_score, int *cand_pos, int *cand_count,
                                  long long cap, void *stream);

/*
 * Stage 3 — sparse MQA attention over the selected latent rows.
 * For row t and head h, over the selected set S_t = {idx[t*k+i] >= 0}:
 *   z_s = softmax_scale * (q[t,h,:] . kv[s,:])   (Dk dims),
 *   out[t,h,:] = sum_s softmax(z)_s * kv[s, 0:Dv],  lse[t,h] = ln sum_s exp(z_s).
 * A row whose S_t is empty gets out = 0 and lse = -inf.
 *   q    device [T][H][Dk] (bf16 or float32: dt)
 *   kv   contiguous: device [B][n_max][Dk]; paged (bf16 only): pool [num_pages][page_size][Dk]
 *   idx  device int32 [T][k]: positions in the row's sequence, -1 = padding;
 *        entries outside 0..pos_t are a device check failure
 *   out  device [T][H][Dv], same dtype as q;  lse device float32 [T][H] or NULL
 *   workspace  device scratch of at least dsa_sparse_mqa_attn_workspace_size() bytes
 *              (256-byte aligned), or NULL when that size is 0
 * Fast path: bf16, H = 128, Dk = 576, Dv = 512, 16-byte aligned rows (tcgen05 MMA).
 * F32: H <= 1024, Dk <= 1024, Dv <= 1024, k <= 8192, contiguous only.
 */
size_t dsa_sparse_mqa_attn_workspace_size(int T, int H, int Dv, int k, dsa_dtype dt);
dsa_status dsa_sparse_mqa_attn(const void *q, const void *kv, dsa_dtype dt,
                               int T, int H, int Dk, int Dv, float softmax_scale,
                               const int *idx, int k, const dsa_seq_layout *lay,
                               void *out, float *lse,
                               void *workspace, size_t ws_bytes, void *stream);

/*
 * Cache write for the decode loop (and prefill chunks): the new token of each query
 * row goes into the caches at the row's own position pos_t (decode: seq_lens[b]-1;
 * prefill: from cu_q), so that the next indexer and attention calls read it.
 * mundobytes.com "Deepseek-v3-2-exp": serving with 64-token KV pages (deployment
 * section) and paged indexer kernels (open-kernels paragraph); jdon.com
 * "DeepSeek-V3.2-Exp": the indexer keys are FP8.
 *   k_new    device [T][d_I] fp32 (k_dt = DSA_F32, 16-byte aligned) or bf16
 *            (DSA_BF16, 8-byte aligned); d_I must be 128. Quantised per token:
 *            scale = max|x| / 448 in fp32 (1 for an all-zero row), code = the e4m3
 *            value nearest to x / scale (IEEE fp32 division), ties to even,
 *            saturating at +-448. Inputs are expected finite.
 *   kv_new   device [T][Dk] bf16 latent rows (16-byte aligned, Dk a multiple of 8,
 *            at most 4096), or NULL to write only the indexer key
 *   lay      the layout the other calls use; it already counts the new token
 *   k_cache  paged (page_size 64): the indexer-key pool, 8448 bytes per page =
 *            [64 x 128 code bytes][64 fp32 scales], k_scale = NULL;
 *            contiguous: [B][n_max][128] code bytes with k_scale [B][n_max] fp32
 *   kv_cache paged: [num_pages*64][Dk] bf16; contiguous: [B][n_max][Dk] bf16
 * Writes only the bytes of each row's own slot. A page id out of range is a
 * device check failure (reported by dsa_get_device_error); rows whose position
 * lies outside the cache are skipped and reported the same way.
 */
dsa_status dsa_cache_append(const void *k_new, dsa_dtype k_dt, const void *kv_new,
                            int T, int d_I, int Dk, const dsa_seq_layout *lay,
                            void *k_cache, float *k_scale, void *kv_cache, void *stream);

/*
 * Indexer training signal on the selected set (sparse stage), loss and gradient.
 * jdon.com "DeepSeek-V3.2-Exp": warm-up paragraph (the indexer is trained to copy the
 * main attention's distribution through a KL-divergence loss, the target being the
 * heads' attention summed and normalised) and sparse-training paragraph (the loss
 * is taken over the selected set; the indexer's gradient is kept apart from the
 * main model's). For row t with S_t = {idx[t*k+i] >= 0}:
 *   p_t(s)   = (1/H) sum_h exp(z_h(s) - lse[t,h]),  z_h(s) = softmax_scale * q[t,h,:] . kv[s,:]
 *   r_t(s)   = exp(scores[t*ld+s]) / sum_{s' in S_t} exp(scores[t*ld+s'])
 *   loss[t]  = sum_{s in S_t} p_t(s) * (ln p_t(s) - ln r_t(s))
 *   grad[t*k+i] = r_t(s_i) - p_t(s_i) = d loss[t] / d scores[t*ld+s_i]  (0 for -1 slots)
 * lse is the attention's log-sum-exp per head over the same S_t, as
 * dsa_sparse_mqa_attn returns it, so that p_t is the heads' mean attention.
 *   q, kv, idx, lay   as for dsa_sparse_mqa_attn (bf16, H = 128, Dk = 576;
 *                     positions in S_t distinct; q and kv 16-byte aligned)
 *   lse      device float32 [T][H];  scores device float32 [T][ld], ld >= the cache extent
 *   loss     device float32 [T] (written: zeroed, then the row's slot ranges add their
 *            terms with atomic adds, so its last bits may differ between runs)
 *   grad     device float32 [T][k], or NULL to skip the gradient
 * idx, lse, scores, loss and grad 4-byte aligned. Index errors are device
 * check failures as in dsa_sparse_mqa_attn; a row with an empty S_t gets loss 0.
 */
dsa_status dsa_indexer_kl(const void *q, const void *kv, dsa_dtype dt,
                          int T, int H, int Dk, float softmax_scale,
                          const int *idx, int k, const dsa_seq_layout *lay,
                          const float *lse, const float *scores, long long ld,
                          float *loss, float *grad, void *stream);

/*
 * Backward of stage 3 for the sparse training stage: gradients of the attention
 * output with respect to the query heads and the selected latent rows.
 * jdon.com "DeepSeek-V3.2-Exp", sparse-training paragraph (the main model is trained
 * on the selected entries only). For row t, head h and s in S_t, with the forward's
 * lse and output o:
 *   P = exp(z - lse[t,h]),  z = softmax_scale * q[t,h,:] . kv[s,:]
 *   dP = dout[t,h,:] . kv[s,0:Dv],  D = dout[t,h,:] . out[t,h,:],  dz = P (dP - D)
 *   dq[t,h,:]  += softmax_scale * sum_s dz kv[s,:]
 *   dkv[s,:]   += softmax_scale * sum_h dz q[t,h,:];  dkv[s,0:Dv] += sum_h P dout[t,h,:]
 * The selection carries no gradient. A position selected by several rows (or twice
 * by one) receives the sum of its slots' contributions.
 *   q, kv, idx, lay   as for dsa_sparse_mqa_attn (bf16, H = 128, Dk = 576, Dv = 512)
 *   out, dout  device bf16 [T][H][Dv]: the forward output and its gradient
 *   lse        device float32 [T][H]: the forward's log-sum-exp
 *   dq         device float32 [T][H][Dk], accumulated into (+=)
 *   dkv        device float32 with the row numbering of kv (contiguous [B][n_max][Dk],
 *              paged [num_pages*page_size][Dk]), accumulated into (+=)
 *   workspace  device scratch of dsa_sparse_mqa_attn_backward_workspace_size(T) bytes,
 *              256-byte aligned
 * Every contribution is an atomic fp32 add, so the last bits of dq and dkv may
 * differ between runs. q, kv, out, dout, dq and dkv 16-byte aligned.
 */
size_t dsa_sparse_mqa_attn_backward_workspace_size(int T);
dsa_status dsa_sparse_mqa_attn_backward(const void *q, const void *kv, dsa_dtype dt,
                                        int T, int H, int Dk, int Dv, float softmax_scale,
                                        const int *idx, int k, const dsa_seq_layout *lay,
                                        const void *out, const void *dout, const float *lse,
                                        float *dq, float *dkv,
                                        void *workspace, size_t ws_bytes, void *stream);

/*
 * Stage 3 without a caller workspace (no counterpart on the pages; this entry
 * point exists for callers, not for the method).
 * Same computation, arguments and dtype as dsa_sparse_mqa_attn with dt = DSA_BF16,
 * minus the workspace: the per-split partial results go to a scratch array of
 * DSA_NOALLOC_SCRATCH_BYTES (40 MiB) that the library owns as a static device
 * variable, so this call never allocates device memory. It is for callers that
 * may not allocate: code running under a host framework that has reserved all
 * device memory up front, or a serving loop where cudaMalloc's implicit device
 * synchronisation is not allowed. The 40 MiB are device memory of the library's
 * module: under CUDA's lazy module loading they are taken when the module is
 * first loaded on a device (at the latest by the first call of this entry point
 * there) and held until the process exits.
 *   - A call needs T * ceil(k/256) * 132096 bytes of scratch (39 decode rows at
 *     k = 2048 fit); larger calls return DSA_ERR_TOO_LARGE and launch nothing.
 *   - The first call on each device looks up the array's device address (with
 *     that device current) and caches it per device index for the life of the
 *     process (the primary context is assumed to live that long: after a
 *     cudaDeviceReset the cached address is stale). Make that first call before
 *     the caller reserves its device memory and before any stream capture. A
 *     call with T = 0 (a prefill layout whose cu_q ranges are all empty) does
 *     only this set-up and launches nothing: a cheap first call.
 *   - All calls share the one array: calls whose kernels may overlap on the GPU
 *     (other streams, other host threads) race on it and must be serialised by
 *     the caller. Nothing in it needs to start at zero.
 * Only DSA_BF16 with H = 128, Dk = 576, Dv = 512 is accepted.
 */
#define DSA_NOALLOC_SCRATCH_BYTES (40ull << 20)
dsa_status dsa_sparse_mqa_attn_noalloc(const void *q, const void *kv, dsa_dtype dt,
                                       int T, int H, int Dk, int Dv, float softmax_scale,
                                       const int *idx, int k, const dsa_seq_layout *lay,
                                       void *out, float *lse, void *stream);

/* All three stages on one stream. */
typedef struct {
  /* indexer */
  const void *q_idx; const float *q_scale;
  const void *k_idx; const float *k_scale;
  dsa_dtype idx_dt; const float *w; int H_I, d_I;
  /* attention */
  const void *q; const void *kv; dsa_dtype attn_dt;
  int H, Dk, Dv; float softmax_scale;
  /* selection and rows */
  int k; int T;
  dsa_seq_layout lay;
  /* outputs */
  void *out; float *lse;          /* lse may be NULL */
  int *idx_out;                   /* optional device int32 [T][k] copy of the selection */
  int topk_path;                  /* how stages 1 and 2 run: DSA_TOPK_AUTO (0, the library's
                                     choice), DSA_TOPK_SCORES (score rows, then dsa_topk) or
                                     DSA_TOPK_FUSED (dsa_indexer_candidates, then
                                     dsa_topk_from_candidates; decode rows with the E4M3 indexer
                                     and a cache capacity up to 262144 keys, else as AUTO) */
} dsa_forward_args;

enum { DSA_TOPK_AUTO = 0, DSA_TOPK_SCORES = 1, DSA_TOPK_FUSED = 2 };

/* Workspace bytes dsa_forward needs for these arguments (0 on invalid arguments). */
size_t dsa_forward_workspace_size(const dsa_forward_args *a);

/*
 * Indexer -> top-k -> attention for a->T rows. a->topk_path picks how the selection
 * is made: score rows then dsa_topk (prefill rows in chunks, so that the score
 * buffer stays within the workspace), or, for decode rows, the fused pair
 * dsa_indexer_candidates + dsa_topk_from_candidates, which writes no score rows.
 * Both give the same selection; DSA_TOPK_AUTO takes the one measured faster on
 * B200 for the shape (today the score rows). The workspace is caller-owned device
 * memory of at least dsa_forward_workspace_size(a) bytes (computed for the same
 * topk_path), 256-byte aligned. No host synchronisation happens inside.
 */
dsa_status dsa_forward(const dsa_forward_args *a, void *workspace, size_t ws_bytes,
                       void *stream);

/* Synchronises `stream`, then returns and clears the device error word:
 * DSA_OK, DSA_ERR_TIMEOUT or DSA_ERR_DEVICE_CHECK (or DSA_ERR_CUDA if the
 * synchronisation itself failed). */
dsa_status dsa_get_device_error(void *stream);

/* As dsa_get_device_error, and also writes (when site != NULL) the code of the
 * first device check or wait that failed (0 when none): a diagnostic for bug
 * reports. */
dsa_status dsa_get_device_error_site(void *stream, unsigned *site);

/* Upper bound, in nanoseconds, of every on-device wait (default 1e9). Applies to
 * launches enqueued after the call. */
dsa_status dsa_set_wait_limit_ns(unsigned long long ns);

const char *dsa_status_string(dsa_status s);
int dsa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DSA_H */
