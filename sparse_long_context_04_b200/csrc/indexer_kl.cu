// Indexer loss on the selected set (sparse stage) and its gradient, on the
// tcgen05 tensor cores.
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
// Work unit (one CTA): row t and up to 256 of its selected slots (fewer when the
// rows alone would leave SMs idle).
//   1. D[256 keys, 128 heads] = K_sel[256, 576] . Q_t[128, 576]^T: the selected
//      latent rows are the M side (two M = 128 tiles, gathered with cp.async into
//      128-byte swizzled tiles), the query's head block the N side (TMA); nine
//      64-dim chunks, tcgen05 kind::f16, fp32 accumulators in TMEM. With the keys
//      on the TMEM lanes, the sum over heads is a sum along one thread's own row.
//   2. Meanwhile the four producer warps, their copies issued, reduce the row's
//      log-sum-exp of the indexer scores over the whole selected set.
//   3. Eight epilogue warps (one key per thread, two per TMEM lane quadrant) form
//      p, r, the gradient and the loss terms; one atomic add per CTA and row.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int kH = 128, kDk = 576;
constexpr int kRowBytes = kDk * 2;             // 1152
constexpr int kKeys = 256;                     // selected slots per CTA
constexpr int kChunks = kDk / 64;              // 9 dim chunks of 128 bytes
constexpr int kStages = 3;
constexpr int kQTile = kH * 128;               // 16 KiB
constexpr int kKTile = kKeys * 128;            // 32 KiB
constexpr int kStage = kQTile + kKTile;        // 48 KiB
constexpr int kRing = kStages * kStage;        // 144 KiB
constexpr int kProducers = 128;                // warps 0-3
constexpr int kMmaWarp = 4;
constexpr int kEpiWarp0 = 5, kEpiWarps = 8;
constexpr int kThreads = 32 * (4 + 1 + kEpiWarps);
constexpr int kSmem = 1024 + kRing + kKeys * 8 + kKeys * 4 + 256;
constexpr int kSplitKeysMin = 64;   // keys per CTA are not split below this
constexpr float kLog2e = 1.4426950408889634f;

struct KlParams {
  const __nv_bfloat16 *kv;
  const int *idx;            // [T][k]
  int k;
  int splits;
  int keys_per_split;        // <= 256
  const float *lse;          // [T][128]
  const float *scores;       // [T][ld]
  long long ld;
  float scale_log2;          // softmax_scale * log2(e)
  float *loss;               // [T], zeroed by the launcher
  float *grad;               // [T][k] or nullptr
  Layout L;
  ErrCtx e;
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void producers_bar() { asm volatile("bar.sync 2, 128;" ::: "memory"); }
__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
// producers publish the row's LSE_I; the epilogue warps wait for it
__device__ __forceinline__ void lse_arrive() { asm volatile("bar.arrive 3, 384;" ::: "memory"); }
__device__ __forceinline__ void lse_wait() { asm volatile("bar.sync 3, 384;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
    indexer_kl_kernel(const __grid_constant__ CUtensorMap tm_q, const KlParams p) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char *base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  unsigned char *ring = base;
  long long *rows = reinterpret_cast<long long *>(base + kRing);
  int *spos = reinterpret_cast<int *>(rows + kKeys);
  uint64_t *bars = reinterpret_cast<uint64_t *>(spos + kKeys);
  // per ring stage: query chunk landed (TMA), key rows landed (cp.async), stage free
  uint64_t *qfull = bars, *kfull = bars + kStages, *empty = bars + 2 * kStages, *s_full = bars + 3 * kStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(s_full + 1);
  __shared__ int s_nvalid;
  __shared__ __align__(16) float s_lse2[kH];   // lse_h * log2(e), read as float2
  __shared__ float s_red[kEpiWarps];
  __shared__ float s_pred[kProducers / 32];
  __shared__ float s_lse_i;

  pdl_prologue();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x / p.splits;
  const int k0 = (blockIdx.x % p.splits) * p.keys_per_split;
  const int nk = min(p.keys_per_split, p.k - k0);
  const int *irow = p.idx + (long long)t * p.k;

  if (threadIdx.x == 0) {
    s_nvalid = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(qfull + s, 1);
      mbar_init(kfull + s, kProducers);
      mbar_init(empty + s, 1);
    }
    mbar_init(s_full, 1);
    fence_mbar_init();
    // the first query chunks do not depend on the selection: start them now
    tma_prefetch_desc(&tm_q);
    for (int c = 0; c < kStages; ++c) {
      mbar_expect_tx(qfull + c, kQTile);
      tma_load_2d(ring + c * kStage, &tm_q, qfull + c, c * 64, t * kH);
    }
  }
  // ---- this CTA's slots (-1 entries are padding, anywhere in the list)
  __syncthreads();
  const RowPos rp = row_position(p.L, t);
  const bool row_ok = rp.len <= cache_capacity(p.L);
  for (int i = threadIdx.x; i < kKeys; i += kThreads) {
    long long r = -1;
    if (i < nk) {
      const int s = __ldg(irow + k0 + i);
      if (s >= 0 && s <= rp.pos && row_ok) {
        r = key_row(p.L, rp.b, s, p.e, 0x700);
      } else if (s != -1) {
        raise_error(p.e, DEV_BOUNDS, 0x701);
      }
      spos[i] = r >= 0 ? s : -1;
    }
    rows[i] = r;
    if (r >= 0) atomicMax(&s_nvalid, i + 1);
  }
  if (threadIdx.x < kH) s_lse2[threadIdx.x] = __ldg(p.lse + (long long)t * kH + threadIdx.x) * kLog2e;
  __syncthreads();
  const int nvalid = s_nvalid;  // entries at or after nvalid are all padding
  if (nvalid == 0) {
    if (p.grad != nullptr && threadIdx.x < nk) p.grad[(long long)t * p.k + k0 + threadIdx.x] = 0.f;
    if (threadIdx.x == 0)  // the early query chunks must land before the CTA exits
      for (int c = 0; c < kStages; ++c) mbar_wait(qfull + c, 0, p.e, 0x702);
    return;
  }
  const int nt = (nvalid + 127) / 128;  // M = 128 key tiles
  const int n = nt * 128;

  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const char *kvb = reinterpret_cast<const char *>(p.kv);

  if (warp < 4) {
    // ================= producers: Q chunks by TMA, selected rows by cp.async
    const int tid = threadIdx.x;
    bool ok = true;
    for (int c = 0; c < kChunks && ok; ++c) {
      const int st = c % kStages;
      ok = mbar_wait(empty + st, ((c / kStages) & 1) ^ 1, p.e, 0x710);
      if (!ok) break;
      unsigned char *sq = ring + st * kStage;
      const uint32_t sk = smem_u32(sq + kQTile);
      if (tid == 0 && c >= kStages) {
        mbar_expect_tx(qfull + st, kQTile);
        tma_load_2d(sq, &tm_q, qfull + st, c * 64, t * kH);
      }
      for (int q = tid; q < n * 8; q += kProducers) {
        const int i = q >> 3, u = q & 7;
        const long long r = rows[i];
        const char *src = kvb + (r >= 0 ? r : 0) * kRowBytes + c * 128 + u * 16;
        cp_async16_zfill(sk + sw128_off(i, u), src, r >= 0);
      }
      cp_async_arrive_noinc(kfull + st);
    }
    // ---- LSE_I over the row's whole selected set, while the copies land
    float mx = -INFINITY;
    for (int j = tid; j < p.k; j += kProducers) {
      const int s = __ldg(irow + j);
      if (s >= 0 && s <= rp.pos) mx = fmaxf(mx, __ldg(p.scores + (long long)t * p.ld + s));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    if (lane == 0) s_pred[warp] = mx;
    producers_bar();
    mx = fmaxf(fmaxf(s_pred[0], s_pred[1]), fmaxf(s_pred[2], s_pred[3]));
    producers_bar();  // all producers have read the maxima
    float se = 0.f;
    for (int j = tid; j < p.k; j += kProducers) {
      const int s = __ldg(irow + j);
      if (s >= 0 && s <= rp.pos) se += ex2_approx((__ldg(p.scores + (long long)t * p.ld + s) - mx) * kLog2e);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) se += __shfl_xor_sync(0xFFFFFFFFu, se, off);
    if (lane == 0) s_pred[warp] = se;
    producers_bar();
    if (tid == 0) s_lse_i = mx + logf((s_pred[0] + s_pred[1]) + (s_pred[2] + s_pred[3]));
    lse_arrive();
    cp_async_wait_all();  // nothing may still land in shared memory after exit
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer: D[keys, heads] += K_sel . Q^T
    if (lane == 0) {
      const uint32_t idesc = instr_desc(1, 1, 0, 0, 128, kH);
      const uint32_t r0 = smem_u32(ring);
      bool ok = true;
      for (int c = 0; c < kChunks && ok; ++c) {
        const int st = c % kStages;
        ok = mbar_wait(qfull + st, (c / kStages) & 1, p.e, 0x720) &&
             mbar_wait(kfull + st, (c / kStages) & 1, p.e, 0x721);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qa = r0 + st * kStage, ka = qa + kQTile;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t bd = smem_desc(qa + ks * 32, 16, 1024, SW_128B);
          for (int m = 0; m < nt; ++m)
            umma_f16(tmem + m * kH, smem_desc(ka + m * 16384 + ks * 32, 16, 1024, SW_128B), bd, idesc,
                     (c | ks) != 0);
        }
        umma_commit(empty + st);
      }
      umma_commit(s_full);
    }
    __syncwarp();
  } else {
    // ================= epilogue: one selected slot per thread
    const int ew = warp - kEpiWarp0;
    const int quad = warp & 3, tile = ew >> 2;
    const int i = tile * 128 + quad * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16) + tile * kH;
    float acc = 0.f;
    bool ok = tile < nt;
    if (ok) ok = mbar_wait(s_full, 0, p.e, 0x730);
    if (ok) {
      tc_fence_after();
      const float2 sc = make_float2(p.scale_log2, p.scale_log2);
      float2 a2 = make_float2(0.f, 0.f);
      for (int j = 0; j < kH / 32; j += 2) {  // two TMEM loads per wait
        uint32_t v[2][32];
        tmem_ld32(trow + j * 32, v[0]);
        tmem_ld32(trow + (j + 1) * 32, v[1]);
        tmem_ld_wait(v[0]);
        tmem_ld_wait(v[1]);
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            const float2 l2 = *reinterpret_cast<const float2 *>(s_lse2 + (j + u) * 32 + x);
            const float2 z = fma2(sc, make_float2(__uint_as_float(v[u][x]), __uint_as_float(v[u][x + 1])),
                                  make_float2(-l2.x, -l2.y));
            a2.x += ex2_approx(z.x);
            a2.y += ex2_approx(z.y);
          }
      }
      acc = a2.x + a2.y;
    }
    const int s = i < nvalid ? spos[i] : -1;
    const bool live = ok && s >= 0;
    const float pj = live ? acc * (1.f / kH) : 0.f;
    lse_wait();
    float c = 0.f, g = 0.f;
    if (live) {
      const float lr = __ldg(p.scores + (long long)t * p.ld + s) - s_lse_i;  // log r
      g = ex2_approx(lr * kLog2e) - pj;
      if (pj > 0.f) c = pj * (logf(pj) - lr);
    }
    if (p.grad != nullptr && i < nk) p.grad[(long long)t * p.k + k0 + i] = g;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, off);
    if (lane == 0) s_red[ew] = c;
    epilogue_bar();
    if (ew == 0 && lane == 0) {
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < kEpiWarps; ++w) tot += s_red[w];
      atomicAdd(p.loss + t, tot);
    }
  }
  if (error_raised(p.e)) {
    // a wait gave up somewhere: copies and MMAs issued before that may still be in flight
    const unsigned long long t0 = globaltimer();
    while (globaltimer() - t0 < 50000ull) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) {
    if (lane == 0) mbar_wait(s_full, 0, p.e, 0x740);
    __syncwarp();
    tmem_dealloc(tmem, 256);
  }
}

__global__ void zero_f32_kernel(float *x, int n) {
  pdl_prologue();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) x[i] = 0.f;
}

}  // namespace

cudaError_t launch_indexer_kl(const void *q, const void *kv, int T, float scale, const int *idx, int k,
                              const float *lse, const float *scores, long long ld, const Layout &L, float *loss,
                              float *grad, const ErrCtx &e, int num_sms, cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(indexer_kl_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (err != cudaSuccess) return err;
  CUtensorMap tq;
  if (!make_q576_map(&tq, q, (unsigned long long)T * kH)) return cudaErrorInvalidValue;
  // fewest splits of at most 256 keys; more (down to 64 keys each) while the rows
  // alone would leave SMs idle
  int splits = (k + kKeys - 1) / kKeys;
  const int fill = num_sms / T;
  const int most = (k + kSplitKeysMin - 1) / kSplitKeysMin;
  if (fill > splits) splits = fill < most ? fill : most;
  const int kps = (k + splits - 1) / splits;
  KlParams p;
  p.kv = static_cast<const __nv_bfloat16 *>(kv);
  p.idx = idx;
  p.k = k;
  p.keys_per_split = kps;
  p.splits = (k + kps - 1) / kps;
  p.lse = lse;
  p.scores = scores;
  p.ld = ld;
  p.scale_log2 = scale * kLog2e;
  p.loss = loss;
  p.grad = grad;
  p.L = L;
  p.e = e;
  err = launch_kernel(zero_f32_kernel, dim3((T + 255) / 256), dim3(256), 0, stream, 0, loss, T);
  if (err != cudaSuccess) return err;
  return launch_kernel(indexer_kl_kernel, dim3((unsigned)T * p.splits), dim3(kThreads), kSmem, stream, 0, tq, p);
}

}  // namespace dsa
