// Backward of the sparse MQA attention over the selected latent rows (dQ, dKV),
// on the tcgen05 tensor cores.
//
// jdon.com "DeepSeek-V3.2-Exp", sparse-training paragraph: the main model is
// trained on the selected entries only (k = 2048 per query token). For row t, head
// h and a selected row s (key = the whole 576-wide row, value = its first 512):
//   P = exp(z - lse_h),  z = scale q_h . kv_s           (the forward's log-sum-exp)
//   dP = dO_h . v_s,  D_h = dO_h . o_h,  dz = P (dP - D_h)
//   dq_h  += scale sum_s dz kv_s
//   dkv_s += scale sum_h dz q_h   (+ sum_h P dO_h on the first 512 dims)
// A position selected by several rows (or slots) accumulates: both outputs are
// fp32 and every contribution is an atomic add.
//
// Work unit (one CTA): row t and 128 of its selected slots. The (Q, dO, K) chunks
// of 64 dims stream twice through one three-stage ring:
//   pass 1  S^T[keys, heads] = K.Q^T and dP^T[keys, heads] = V.dO^T: the gathered
//           rows are the M = 128 side (cp.async into 128-byte swizzled tiles), the
//           query and output-gradient head blocks the N = 128 side (TMA); fp32 in
//           TMEM.
//   then    eight warps turn each (key, head) into P and scale*dz, stored as bf16
//           tiles in shared memory: one row per key, 64 heads per 128-byte row.
//   pass 2  per 64-dim chunk c: dKV_c[keys, 64] = dZ^T.Q_c + P^T.dO_c (A K-major,
//           B MN-major) and dQ_c[heads, 64] = dZ.K_c (the same dZ tile read
//           MN-major as A, the key tile MN-major as B), double-buffered in TMEM;
//           four warps add dKV_c into the selected rows, four add dQ_c into dq.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int kH = 128, kDk = 576, kDv = 512;
constexpr int kRowBytes = kDk * 2;             // 1152
constexpr int kKeys = 128;                     // selected slots per CTA
constexpr int kChunks = kDk / 64;              // 9 dim chunks of 128 bytes
constexpr int kVChunks = kDv / 64;             // 8 of them are value dims
constexpr int kLoads = 2 * kChunks;            // each chunk streams once per pass
constexpr int kStages = 3;
constexpr int kTile = 128 * 128;               // 16 KiB: 128 rows x 128 bytes
constexpr int kStage = 3 * kTile;              // Q_c, dO_c, K_c
constexpr int kRing = kStages * kStage;        // 144 KiB
constexpr int kHalfTile = 2 * kTile;           // dZ or P: two 64-head groups
constexpr int kProducers = 128;                // warps 0-3
constexpr int kMmaWarp = 4;
constexpr int kEpiWarp0 = 5, kEpiWarps = 8;
constexpr int kThreads = 32 * (4 + 1 + kEpiWarps);
constexpr int kSmem = 1024 + kRing + 2 * kHalfTile + kKeys * 8 + 256;
constexpr float kLog2e = 1.4426950408889634f;
// TMEM columns: pass 1 S^T at 0 and dP^T at 128; pass 2 dKV buffers at 0 and 64,
// dQ buffers at 128 and 192
constexpr uint32_t kColDP = 128, kColDQ = 128;

struct BwdParams {
  const __nv_bfloat16 *kv;
  const int *idx;      // [T][k]
  int k;
  int splits;
  const float *lse;    // [T][128], the forward's
  const float *delta;  // [T][128], dO . o per head
  float scale;
  float scale_log2;    // scale * log2(e)
  float *dq;           // [T][128][576] fp32, accumulated
  float *dkv;          // rows of 576 fp32 (same row numbering as kv), accumulated
  Layout L;
  ErrCtx e;
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char *base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  unsigned char *ring = base;
  unsigned char *sZ = base + kRing;         // scale*dz as bf16: [head group][key][64 heads], swizzled
  unsigned char *sP = sZ + kHalfTile;       // P as bf16, same layout
  long long *rows = reinterpret_cast<long long *>(sP + kHalfTile);
  uint64_t *bars = reinterpret_cast<uint64_t *>(rows + kKeys);
  uint64_t *qfull = bars, *kfull = bars + kStages, *empty = bars + 2 * kStages;
  uint64_t *s_full = bars + 3 * kStages, *p_full = s_full + 1, *done = p_full + 1;
  uint64_t *acc_full = done + 1, *acc_empty = acc_full + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
  __shared__ int s_nvalid;
  __shared__ float s_lse2[kH];  // lse_h * log2(e)
  __shared__ float s_delta[kH];

  pdl_prologue();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x / p.splits;
  const int k0 = (blockIdx.x % p.splits) * kKeys;
  const int nk = min(kKeys, p.k - k0);

  // ---- this CTA's slots (-1 entries are padding, anywhere in the list)
  if (threadIdx.x == 0) s_nvalid = 0;
  __syncthreads();
  const RowPos rp = row_position(p.L, t);
  const bool row_ok = rp.len <= cache_capacity(p.L);
  for (int i = threadIdx.x; i < kKeys; i += kThreads) {
    long long r = -1;
    if (i < nk) {
      const int s = __ldg(p.idx + (long long)t * p.k + k0 + i);
      if (s >= 0 && s <= rp.pos && row_ok) {
        r = key_row(p.L, rp.b, s, p.e, 0x800);
      } else if (s != -1) {
        raise_error(p.e, DEV_BOUNDS, 0x801);
      }
    }
    rows[i] = r;
    if (r >= 0) atomicMax(&s_nvalid, i + 1);
  }
  if (threadIdx.x < kH) {
    s_lse2[threadIdx.x] = __ldg(p.lse + (long long)t * kH + threadIdx.x) * kLog2e;
    s_delta[threadIdx.x] = __ldg(p.delta + (long long)t * kH + threadIdx.x);
  }
  __syncthreads();
  const int nvalid = s_nvalid;
  if (nvalid == 0) return;  // nothing selected here: no contribution

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(qfull + s, 1);
      mbar_init(kfull + s, kProducers);
      mbar_init(empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, kEpiWarps);
    mbar_init(done, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, kEpiWarps);
    }
    fence_mbar_init();
  }
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
    // ================= producers: Q_c and dO_c by TMA, the selected rows' chunk c by cp.async
    const int tid = threadIdx.x;
    if (tid == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
    }
    bool ok = true;
    for (int l = 0; l < kLoads && ok; ++l) {
      const int c = l % kChunks, st = l % kStages;
      ok = mbar_wait(empty + st, ((l / kStages) & 1) ^ 1, p.e, 0x810);
      if (!ok) break;
      unsigned char *sq = ring + st * kStage;
      const uint32_t sk = smem_u32(sq + 2 * kTile);
      if (tid == 0) {
        mbar_expect_tx(qfull + st, c < kVChunks ? 2 * kTile : kTile);
        tma_load_2d(sq, &tm_q, qfull + st, c * 64, t * kH);
        if (c < kVChunks) tma_load_2d(sq + kTile, &tm_do, qfull + st, c * 64, t * kH);
      }
      for (int q = tid; q < kKeys * 8; q += kProducers) {
        const int i = q >> 3, u = q & 7;
        const long long r = rows[i];
        const char *src = kvb + (r >= 0 ? r : 0) * kRowBytes + c * 128 + u * 16;
        cp_async16_zfill(sk + sw128_off(i, u), src, r >= 0);
      }
      cp_async_arrive_noinc(kfull + st);
    }
    cp_async_wait_all();  // nothing may still land in shared memory after exit
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = instr_desc(1, 1, 0, 0, 128, kH);   // keys x heads, both K-major
      const uint32_t idesc_kv = instr_desc(1, 1, 0, 1, 128, 64);  // keys x 64 dims over heads
      const uint32_t idesc_q = instr_desc(1, 1, 1, 1, 128, 64);   // heads x 64 dims over keys
      const uint32_t r0 = smem_u32(ring), z0 = smem_u32(sZ), p0 = smem_u32(sP);
      bool ok = true;
      // pass 1: S^T and dP^T over the nine chunks
      for (int l = 0; l < kChunks && ok; ++l) {
        const int st = l % kStages, ph = (l / kStages) & 1;
        ok = mbar_wait(qfull + st, ph, p.e, 0x820) && mbar_wait(kfull + st, ph, p.e, 0x821);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qa = r0 + st * kStage, da = qa + kTile, ka = da + kTile;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = smem_desc(ka + ks * 32, 16, 1024, SW_128B);
          umma_f16(tmem, ad, smem_desc(qa + ks * 32, 16, 1024, SW_128B), idesc_s, (l | ks) != 0);
          if (l < kVChunks)
            umma_f16(tmem + kColDP, ad, smem_desc(da + ks * 32, 16, 1024, SW_128B), idesc_s, (l | ks) != 0);
        }
        umma_commit(empty + st);
      }
      umma_commit(s_full);
      if (ok) ok = mbar_wait(p_full, 0, p.e, 0x822);
      if (ok) tc_fence_after();
      // pass 2: dKV_c and dQ_c per chunk
      for (int c = 0; c < kChunks && ok; ++c) {
        const int l = kChunks + c, st = l % kStages, ph = (l / kStages) & 1;
        const int b = c & 1;
        ok = mbar_wait(qfull + st, ph, p.e, 0x823) && mbar_wait(kfull + st, ph, p.e, 0x824) &&
             mbar_wait(acc_empty + b, ((c >> 1) & 1) ^ 1, p.e, 0x825);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qa = r0 + st * kStage, da = qa + kTile, ka = da + kTile;
        const uint32_t dkv_acc = tmem + b * 64, dq_acc = tmem + kColDQ + b * 64;
        // dKV_c[keys, 64] = dZ^T[keys, heads] . Q_c[heads, 64] (+ P^T . dO_c): 16 heads per step
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_f16(dkv_acc, smem_desc(z0 + (ks >> 2) * kTile + (ks & 3) * 32, 16, 1024, SW_128B),
                   smem_desc(qa + ks * 2048, kTile, 1024, SW_128B), idesc_kv, ks != 0);
        if (c < kVChunks) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            umma_f16(dkv_acc, smem_desc(p0 + (ks >> 2) * kTile + (ks & 3) * 32, 16, 1024, SW_128B),
                     smem_desc(da + ks * 2048, kTile, 1024, SW_128B), idesc_kv, 1);
        }
        // dQ_c[heads, 64] = dZ[heads, keys] . K_c[keys, 64]: 16 keys per step; the dZ
        // tile read MN-major (heads contiguous, the two 64-head groups kTile apart)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_f16(dq_acc, smem_desc(z0 + ks * 2048, kTile, 1024, SW_128B),
                   smem_desc(ka + ks * 2048, kTile, 1024, SW_128B), idesc_q, ks != 0);
        umma_commit(empty + st);
        umma_commit(acc_full + b);
      }
      umma_commit(done);
    }
    __syncwarp();
  } else {
    // ================= epilogue warps
    const int ew = warp - kEpiWarp0;
    const int quad = warp & 3;
    const int j = quad * 32 + lane;  // TMEM lane: a key in pass 1 and dKV, a head in dQ
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const bool live = j < nvalid && rows[j] >= 0;
    bool ok = mbar_wait(s_full, 0, p.e, 0x830);
    if (ok) {
      // P and scale*dz for key j and the 64 heads of group hg, 32 heads per round
      tc_fence_after();
      const int hg = ew >> 2;
      unsigned char *zrow = sZ + hg * kTile, *prow = sP + hg * kTile;
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int h0 = hg * 64 + x * 32;
        uint32_t vs[32], vd[32];
        tmem_ld32(trow + h0, vs);
        tmem_ld32(trow + kColDP + h0, vd);
        tmem_ld_wait(vs);
        tmem_ld_wait(vd);
        uint32_t pz[16], pp[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float P0 = 0.f, P1 = 0.f;
          if (live) {
            P0 = ex2_approx(fmaf(__uint_as_float(vs[i]), p.scale_log2, -s_lse2[h0 + i]));
            P1 = ex2_approx(fmaf(__uint_as_float(vs[i + 1]), p.scale_log2, -s_lse2[h0 + i + 1]));
          }
          const float z0v = P0 * (__uint_as_float(vd[i]) - s_delta[h0 + i]) * p.scale;
          const float z1v = P1 * (__uint_as_float(vd[i + 1]) - s_delta[h0 + i + 1]) * p.scale;
          pp[i >> 1] = pack_bf16(P0, P1);
          pz[i >> 1] = pack_bf16(z0v, z1v);
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const uint32_t off = sw128_off((uint32_t)j, (uint32_t)(x * 4 + c4));
          *reinterpret_cast<uint4 *>(zrow + off) = make_uint4(pz[c4 * 4], pz[c4 * 4 + 1], pz[c4 * 4 + 2], pz[c4 * 4 + 3]);
          *reinterpret_cast<uint4 *>(prow + off) = make_uint4(pp[c4 * 4], pp[c4 * 4 + 1], pp[c4 * 4 + 2], pp[c4 * 4 + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // pass 2: warps 5-8 add dKV rows (lane = key), warps 9-12 add dQ rows (lane = head)
    const bool kv_side = ew < 4;
    float *dst_row = kv_side ? (live ? p.dkv + rows[j] * kDk : nullptr)
                             : p.dq + ((long long)t * kH + j) * kDk;
    for (int c = 0; c < kChunks && ok; ++c) {
      const int b = c & 1;
      ok = mbar_wait(acc_full + b, (c >> 1) & 1, p.e, 0x840);
      if (!ok) break;
      tc_fence_after();
      uint32_t v[2][32];
      const uint32_t col = (kv_side ? 0u : kColDQ) + b * 64;
      tmem_ld32(trow + col, v[0]);
      tmem_ld32(trow + col + 32, v[1]);
      tmem_ld_wait(v[0]);
      tmem_ld_wait(v[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + b);  // the buffer may be overwritten now
      if (dst_row != nullptr) {
        float4 *dst = reinterpret_cast<float4 *>(dst_row + c * 64);
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            atomicAdd(dst + u * 8 + q, make_float4(__uint_as_float(v[u][q * 4]), __uint_as_float(v[u][q * 4 + 1]),
                                                   __uint_as_float(v[u][q * 4 + 2]),
                                                   __uint_as_float(v[u][q * 4 + 3])));
      }
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
    if (lane == 0) mbar_wait(done, 0, p.e, 0x850);
    __syncwarp();
    tmem_dealloc(tmem, 256);
  }
}

// D[t][h] = dO[t,h,:] . o[t,h,:] over the 512 value dims: one warp per (row, head)
__global__ void __launch_bounds__(256) attn_bwd_delta_kernel(const __nv_bfloat16 *__restrict__ out,
                                                             const __nv_bfloat16 *__restrict__ dout, int n,
                                                             float *__restrict__ delta) {
  pdl_prologue();
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (w >= n) return;
  const uint4 *o = reinterpret_cast<const uint4 *>(out + (long long)w * kDv);
  const uint4 *d = reinterpret_cast<const uint4 *>(dout + (long long)w * kDv);
  float acc = 0.f;
#pragma unroll
  for (int i = lane; i < kDv / 8; i += 32) {
    const uint4 a = __ldg(o + i), g = __ldg(d + i);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&av[u]));
      const float2 fg = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&gv[u]));
      acc = fmaf(fa.x, fg.x, fmaf(fa.y, fg.y, acc));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
  if (lane == 0) delta[w] = acc;
}

}  // namespace

size_t attn_bwd_workspace(int T) { return ((size_t)T * kH * sizeof(float) + 255) & ~size_t(255); }

cudaError_t launch_attn_bwd(const void *q, const void *kv, int T, float scale, const int *idx, int k,
                            const Layout &L, const void *out, const void *dout, const float *lse, float *dq,
                            float *dkv, void *ws, const ErrCtx &e, cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(attn_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (err != cudaSuccess) return err;
  CUtensorMap tq, tdo;
  if (!make_bf16_rows_map(&tq, q, (unsigned long long)T * kH, kDk)) return cudaErrorInvalidValue;
  if (!make_bf16_rows_map(&tdo, dout, (unsigned long long)T * kH, kDv)) return cudaErrorInvalidValue;
  float *delta = static_cast<float *>(ws);
  const int n = T * kH;
  err = launch_kernel(attn_bwd_delta_kernel, dim3((n + 7) / 8), dim3(256), 0, stream, 0,
                      static_cast<const __nv_bfloat16 *>(out), static_cast<const __nv_bfloat16 *>(dout), n, delta);
  if (err != cudaSuccess) return err;
  BwdParams p;
  p.kv = static_cast<const __nv_bfloat16 *>(kv);
  p.idx = idx;
  p.k = k;
  p.splits = (k + kKeys - 1) / kKeys;
  p.lse = lse;
  p.delta = delta;
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.dq = dq;
  p.dkv = dkv;
  p.L = L;
  p.e = e;
  return launch_kernel(attn_bwd_kernel, dim3((unsigned)T * p.splits), dim3(kThreads), kSmem, stream, 0, tq, tdo, p);
}

}  // namespace dsa
