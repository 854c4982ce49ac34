// Sparse MQA attention over the selected latent rows on the tcgen05 tensor cores.
//
// jdon.com "DeepSeek-V3.2-Exp", selection paragraph: only the k chosen key/value
// entries take part in attention; openi.cn "DeepSeek-V3.2", MLA-in-MQA-mode item:
// one latent entry is shared by every query head. Each selected row is 576 bf16
// values; the key is the whole row, the value its first 512 values.
//
// Work unit (one CTA): query row t and a split of up to 256 of its selected
// positions. One pass, no running rescale:
//   1. S[128 heads, n] = Q_t[128, 576] . K_sel[n, 576]^T  — nine 64-dim chunks,
//      Q by a tiled TMA load and the selected rows by TMA four-row gathers into
//      128-byte swizzled tiles; tcgen05 kind::f16, M = 128, N = n, in TMEM.
//   2. Four warps (one head row per thread) read S from TMEM, take the row max
//      and write P = exp(scale (S - max)) as bf16 into shared memory.
//   3. O[128, 512] = P[128, n] . V[n, 512] with the value rows gathered again
//      (MN-major B operand, same tile shape); O reuses the TMEM columns S occupied.
//   4. O, normalised by the split's own sum, is staged as fp16 in the freed score
//      ring and leaves with bulk stores; the row max and sum go beside it. A
//      second kernel merges the splits of each row with log-sum-exp weights.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <mutex>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int kH = 128, kDk = 576, kDv = 512;
constexpr int kRowBytes = kDk * 2;   // 1152
constexpr int kMaxKeys = 256;        // keys per split
constexpr int kChunks = kDk / 64;    // 9 dim chunks of 128 bytes
constexpr int kStages = 3;
constexpr int kQTile = kH * 128;               // 16 KiB
constexpr int kKTile = kMaxKeys * 128;         // 32 KiB
constexpr int kStage = kQTile + kKTile;        // 48 KiB
constexpr int kRing = kStages * kStage;        // 144 KiB (later: four 32 KiB value blocks)
constexpr int kVKeys = 32;                     // value rows per block
constexpr int kVBlock = kVKeys * kDv * 2;      // 32 KiB
constexpr int kVStages = 4;
constexpr int kPBytes = kH * kMaxKeys * 2;     // 64 KiB
constexpr int kProducerWarps = 4;              // warps 0-3
constexpr int kMmaWarp = 4;
constexpr int kSmWarp0 = 5, kSmWarps = 8;      // softmax/output warps: two per TMEM lane quadrant
constexpr int kThreads = 32 * (4 + 1 + kSmWarps);
constexpr int kSmem = 1024 + kRing + kPBytes + kMaxKeys * 4 + 256 + 1024;
constexpr int kRowsPerLaunch = 296;            // bounds the partial-result workspace
constexpr int kSlice = kH * 128;               // staged output of 64 values of all heads (fp16)
static_assert((kDv / 64) * kSlice <= kRing, "the staged output reuses the score ring");
static_assert(kVStages * kVBlock <= kRing, "value blocks reuse the score ring");

struct Params {
  int kv_rows;        // rows of the latent cache; the gather coordinate of a padding entry
  const int *idx;
  int k;
  int splits;
  int keys_per_split;
  float scale_log2;   // softmax_scale * log2(e)
  float scale;
  __half *o_part;     // [rows][splits][8 chunks of 64 values][128 heads][64 values]: each
                      // split's output normalised by its own softmax sum; the 16-byte
                      // pieces of a head's 64 values are swizzled (piece ^ (head & 7))
  float2 *ml_part;    // [rows][splits][128]: (max * scale, sum)
  Layout L;
  ErrCtx e;
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}

// 2^x by the MUFU approximation (relative error ~2^-22, far below the bf16 rounding of P)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// the eight softmax/output warps only
__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_half(float a, float b) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                     const Params p) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char *base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  unsigned char *ring = base;
  unsigned char *sP = base + kRing;
  int *rows = reinterpret_cast<int *>(sP + kPBytes);  // gather row of each selected entry
  uint64_t *bars = reinterpret_cast<uint64_t *>(rows + kMaxKeys);
  uint64_t *full = bars, *empty = bars + kStages;
  uint64_t *vfull = bars + 2 * kStages, *vempty = vfull + kVStages;
  uint64_t *s_full = vempty + kVStages, *p_full = s_full + 1, *o_full = p_full + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(o_full + 1);
  __shared__ int s_nvalid;
  __shared__ uint32_t s_valid[kMaxKeys / 32];  // bit i: selected entry i is a real row
  __shared__ float s_part[2][kH];              // per-half row max, then row sum

  pdl_prologue();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x / p.splits;     // row within this launch
  const int split = blockIdx.x % p.splits;
  const int k0 = split * p.keys_per_split;
  const int nk = min(p.keys_per_split, p.k - k0);
  const long long part = (long long)t * p.splits + split;

  // ---- selected rows of this split (-1 entries are padding, anywhere in the list)
  if (threadIdx.x == 0) s_nvalid = 0;
  if (threadIdx.x < kMaxKeys / 32) s_valid[threadIdx.x] = 0;
  __syncthreads();
  const RowPos rp = row_position(p.L, t);
  for (int i = threadIdx.x; i < kMaxKeys; i += kThreads) {
    long long r = -1;
    if (i < nk) {
      const int s = __ldg(p.idx + (long long)t * p.k + k0 + i);
      if (s >= 0 && s <= rp.pos && rp.len <= cache_capacity(p.L)) {
        r = key_row(p.L, rp.b, s, p.e, 0x500);
      } else if (s != -1) {
        raise_error(p.e, DEV_BOUNDS, 0x501);
      }
    }
    rows[i] = r >= 0 ? (int)r : p.kv_rows;  // padding reads the zero fill past the last row
    if (r >= 0) {
      atomicMax(&s_nvalid, i + 1);
      atomicOr(&s_valid[i >> 5], 1u << (i & 31));
    }
  }
  __syncthreads();
  const int nvalid = s_nvalid;  // entries at or after nvalid are all padding
  if (nvalid == 0) {
    if (threadIdx.x < kH) p.ml_part[part * kH + threadIdx.x] = make_float2(-INFINITY, 0.f);
    return;
  }
  const int n = ((nvalid + 63) / 64) * 64;  // MMA N of the score tile
  const int nvb = (nvalid + kVKeys - 1) / kVKeys;  // value blocks

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, kProducerWarps);
      mbar_init(empty + s, 1);
    }
    for (int j = 0; j < kVStages; ++j) {
      mbar_init(vfull + j, kProducerWarps);
      mbar_init(vempty + j, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, kSmWarps);
    mbar_init(o_full, 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < kProducerWarps) {
    // ================= producers: Q chunks by a tiled TMA load, selected rows by
    // four-row TMA gathers. Warp w's lanes issue the row groups g = 4 * lane + w, after
    // lane 0 has announced the warp's bytes on the stage barrier.
    const int tid = threadIdx.x;
    if (tid == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_kv);
    }
    const int groups = n / 16;  // row groups per warp and chunk (n is a multiple of 64)
    bool ok = true;
    for (int c = 0; c < kChunks && ok; ++c) {
      const int st = c % kStages;
      ok = mbar_wait(empty + st, ((c / kStages) & 1) ^ 1, p.e, 0x510);
      if (!ok) break;
      unsigned char *sq = ring + st * kStage;
      unsigned char *sk = sq + kQTile;
      if (lane == 0) mbar_expect_tx(full + st, groups * 512 + (warp == 0 ? kQTile : 0));
      __syncwarp();
      if (tid == 0) tma_load_2d(sq, &tm_q, full + st, c * 64, t * kH);
      if (lane < groups) {
        const int g = 4 * lane + warp;  // keys 4g .. 4g+3: rows 4g .. 4g+3 of the chunk's tile
        tma_gather4(sk + g * 512, &tm_kv, full + st, c * 64, rows[4 * g], rows[4 * g + 1], rows[4 * g + 2],
                    rows[4 * g + 3]);
      }
    }
    // value rows: wait until every score MMA has consumed the ring
    if (ok) ok = mbar_wait(s_full, 0, p.e, 0x511);
    for (int vb = 0; vb < nvb && ok; ++vb) {
      const int st = vb % kVStages;
      ok = mbar_wait(vempty + st, ((vb / kVStages) & 1) ^ 1, p.e, 0x512);
      if (!ok) break;
      // 32 value rows x 8 dim chunks: 64 gathers, 16 per warp; chunk u of the block is
      // a [32 rows x 128 bytes] tile
      unsigned char *sv = ring + st * kVBlock;
      if (lane == 0) mbar_expect_tx(vfull + st, 16 * 512);
      __syncwarp();
      if (lane < 16) {
        const int q = 4 * lane + warp, u = q >> 3, g = q & 7;
        const int *rg = rows + vb * kVKeys + 4 * g;
        tma_gather4(sv + u * (kVKeys * 128) + g * 512, &tm_kv, vfull + st, u * 64, rg[0], rg[1], rg[2], rg[3]);
      }
    }
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = instr_desc(1, 1, 0, 0, 128, (uint32_t)n);
      const uint32_t idesc_pv = instr_desc(1, 1, 0, 1, 128, 256);
      const uint32_t r0 = smem_u32(ring), p0 = smem_u32(sP);
      bool ok = true;
      for (int c = 0; c < kChunks && ok; ++c) {
        const int st = c % kStages;
        ok = mbar_wait(full + st, (c / kStages) & 1, p.e, 0x520);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qa = r0 + st * kStage, ka = qa + kQTile;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_f16(tmem, smem_desc(qa + ks * 32, 16, 1024, SW_128B), smem_desc(ka + ks * 32, 16, 1024, SW_128B),
                   idesc_qk, (c | ks) != 0);
        umma_commit(empty + st);
      }
      umma_commit(s_full);
      if (ok) ok = mbar_wait(p_full, 0, p.e, 0x521);
      if (ok) tc_fence_after();
      for (int vb = 0; vb < nvb && ok; ++vb) {
        const int st = vb % kVStages;
        ok = mbar_wait(vfull + st, (vb / kVStages) & 1, p.e, 0x522);
        if (!ok) break;
        tc_fence_after();
        // value rows vb*32 .. +31: their P columns sit in 64-key block vb/2, bytes (vb%2)*64 of each row
        const uint32_t va = r0 + st * kVBlock, pa = p0 + (vb >> 1) * 16384 + (vb & 1) * 64;
#pragma unroll
        for (int ks = 0; ks < kVKeys / 16; ++ks) {
          const uint64_t ad = smem_desc(pa + ks * 32, 16, 1024, SW_128B);
#pragma unroll
          for (int nh = 0; nh < 2; ++nh)
            umma_f16(tmem + nh * 256, ad,
                     smem_desc(va + nh * 4 * (kVKeys * 128) + ks * 2048, kVKeys * 128, 1024, SW_128B), idesc_pv,
                     (vb | ks) != 0);
        }
        umma_commit(vempty + st);
      }
      umma_commit(o_full);
    }
    __syncwarp();
  } else {
    // ================= softmax + output: 8 warps, two per TMEM lane quadrant, each half the columns
    const int sw = warp - kSmWarp0;
    const int quad = warp & 3;
    const int half = sw >> 2;
    const int h = quad * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const int j0 = half * (n / 64), j1 = j0 + n / 64;  // this half's 32-column chunks
    float m = -INFINITY, l = 0.f;
    bool ok = mbar_wait(s_full, 0, p.e, 0x530);
    if (ok) {
      tc_fence_after();
      for (int j = j0; j < j1; j += 2) {  // two TMEM loads per wait
        uint32_t v[2][32];
        tmem_ld32(trow + j * 32, v[0]);
        if (j + 1 < j1) tmem_ld32(trow + (j + 1) * 32, v[1]);
        tmem_ld_wait(v[0]);
        tmem_ld_wait(v[1]);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (j + u >= j1) break;
          const uint32_t vm = s_valid[j + u];
#pragma unroll
          for (int x = 0; x < 32; ++x)
            if ((vm >> x) & 1u) m = fmaxf(m, __uint_as_float(v[u][x]));
        }
      }
    }
    s_part[half][h] = m;
    softmax_bar();
    m = fmaxf(s_part[0][h], s_part[1][h]);
    softmax_bar();  // both halves have read the maxima
    const float mb = m * p.scale_log2;
    if (ok) {
      for (int j = j0; j < j1; ++j) {
        uint32_t v[32];
        tmem_ld32(trow + j * 32, v);
        tmem_ld_wait(v);
        const uint32_t vm = s_valid[j];
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float2 z = fma2(make_float2(p.scale_log2, p.scale_log2),
                                make_float2(__uint_as_float(v[x]), __uint_as_float(v[x + 1])), make_float2(-mb, -mb));
          const float a = ((vm >> x) & 1u) ? ex2_approx(z.x) : 0.f;
          const float b = ((vm >> (x + 1)) & 1u) ? ex2_approx(z.y) : 0.f;
          const uint32_t w = pack_bf16(a, b);
          pk[x >> 1] = w;
          __nv_bfloat162 bw = *reinterpret_cast<const __nv_bfloat162 *>(&w);
          l += __low2float(bw) + __high2float(bw);
        }
        // keys j*32 .. j*32+31 sit in 64-key block j/2, 16-byte chunks (j%2)*4 .. +3
        unsigned char *pb = sP + (j >> 1) * 16384;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const uint32_t off = sw128_off((uint32_t)h, (uint32_t)((j & 1) * 4 + c4));
          *reinterpret_cast<uint4 *>(pb + off) = make_uint4(pk[c4 * 4], pk[c4 * 4 + 1], pk[c4 * 4 + 2], pk[c4 * 4 + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    s_part[half][h] = l;
    softmax_bar();
    l = s_part[0][h] + s_part[1][h];
    if (ok) ok = mbar_wait(o_full, 0, p.e, 0x531);
    if (ok) {
      tc_fence_after();
      // this warp's 256 output columns, normalised by the split's own sum: a convex
      // combination of value rows, so fp16 keeps ~1e-3 absolute accuracy. Staged in the
      // score ring (all its loads have been consumed by now) in the workspace's layout.
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      for (int j = half * 8; j < half * 8 + 8; j += 2) {
        uint32_t v[2][32];
        tmem_ld32(trow + j * 32, v[0]);
        tmem_ld32(trow + (j + 1) * 32, v[1]);
        tmem_ld_wait(v[0]);
        tmem_ld_wait(v[1]);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          unsigned char *cb = ring + ((j + u) >> 1) * kSlice + h * 128;  // values 32(j+u) .. +31
#pragma unroll
          for (int pc = 0; pc < 4; ++pc) {
            uint32_t w[4];
#pragma unroll
            for (int y = 0; y < 4; ++y)
              w[y] = pack_half(__uint_as_float(v[u][pc * 8 + 2 * y]) * inv_l,
                               __uint_as_float(v[u][pc * 8 + 2 * y + 1]) * inv_l);
            const int piece = ((j + u) & 1) * 4 + pc;
            *reinterpret_cast<uint4 *>(cb + ((piece ^ (h & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      fence_proxy_async_smem();
      if (half == 0) p.ml_part[part * kH + h] = make_float2(m * p.scale, l);
    } else if (half == 0) {
      p.ml_part[part * kH + h] = make_float2(-INFINITY, 0.f);
    }
    softmax_bar();  // the whole output tile is staged
    if (ok && sw == 0 && lane == 0) {
      char *dst = reinterpret_cast<char *>(p.o_part + part * (long long)(kDv * kH));
      for (int c = 0; c < kDv / 64; ++c) bulk_store(dst + c * kSlice, ring + c * kSlice, kSlice);
      bulk_commit();
      bulk_wait_read_all();  // the staged tile is read before this CTA ends
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
    // all MMAs have completed once o_full fired; if a wait gave up, wait here (bounded)
    if (lane == 0) mbar_wait(o_full, 0, p.e, 0x540);
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the splits of each (row, head). One thread per 16-byte piece of the
// output (8 values of one head), 128 per CTA, eight CTAs per 64-value chunk of a
// row. With O_c the split's output already divided by its sum l_c and M the
// largest max of the head over the splits that hold keys:
// out = sum_c (e^{m_c - M} l_c) O_c / sum_c e^{m_c - M} l_c, lse = M + ln(denominator).
// Each thread forms the weights of its head itself, so that the (max, sum) pairs
// and the pieces of up to eight splits are all in flight at once.
constexpr int kCombThreads = 128;  // small CTAs: a decode batch's grid fills the GPU in one wave
constexpr int kCombPer = (kSlice / 16) / kCombThreads;  // CTAs per 64-value chunk of a row
constexpr int kCombSplits = 8;                          // splits loaded together
__global__ void __launch_bounds__(kCombThreads)
    attn_combine_kernel(const __half *__restrict__ o_part, const float2 *__restrict__ ml_part, int splits,
                        __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
  pdl_prologue();
  const int t = blockIdx.x, ch = blockIdx.y / kCombPer;
  const int q = (blockIdx.y % kCombPer) * kCombThreads + threadIdx.x, h = q >> 3, piece = q & 7;
  const float2 *ml = ml_part + (long long)t * splits * kH + h;
  const char *ob = reinterpret_cast<const char *>(o_part + (long long)t * splits * (kDv * kH)) + ch * kSlice +
                   h * 128 + ((piece ^ (h & 7)) << 4);
  constexpr long long kSplitBytes = (long long)kDv * kH * 2;
  float M = -INFINITY, L = 0.f;
  float acc[8];
#pragma unroll
  for (int x = 0; x < 8; ++x) acc[x] = 0.f;
  // the running max M changes only between groups of eight splits: the accumulated
  // sums are rescaled when it does (exactly the single-pass result when splits <= 8)
  for (int c0 = 0; c0 < splits; c0 += kCombSplits) {
    float2 v[kCombSplits];
    uint4 r[kCombSplits];
#pragma unroll
    for (int u = 0; u < kCombSplits; ++u) {
      const int c = c0 + u;
      v[u] = c < splits ? ml[c * kH] : make_float2(-INFINITY, 0.f);
      if (c < splits) r[u] = __ldcs(reinterpret_cast<const uint4 *>(ob + c * kSplitBytes));
    }
    float Mn = M;
#pragma unroll
    for (int u = 0; u < kCombSplits; ++u)
      if (v[u].y > 0.f) Mn = fmaxf(Mn, v[u].x);
    if (Mn != M && M != -INFINITY) {
      const float f = __expf(M - Mn);
      L *= f;
#pragma unroll
      for (int x = 0; x < 8; ++x) acc[x] *= f;
    }
    M = Mn;
#pragma unroll
    for (int u = 0; u < kCombSplits; ++u) {
      // a split without keys wrote no output: its weight is 0 and its piece is not read
      const float w = v[u].y > 0.f ? __expf(v[u].x - M) * v[u].y : 0.f;
      L += w;
      if (w == 0.f) continue;
      const __half2 *hv = reinterpret_cast<const __half2 *>(&r[u]);
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        const float2 f = __half22float2(hv[y]);
        acc[2 * y] = fmaf(w, f.x, acc[2 * y]);
        acc[2 * y + 1] = fmaf(w, f.y, acc[2 * y + 1]);
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  *reinterpret_cast<uint4 *>(out + ((long long)t * kH + h) * kDv + ch * 64 + piece * 8) =
      make_uint4(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv),
                 pack_bf16(acc[4] * inv, acc[5] * inv), pack_bf16(acc[6] * inv, acc[7] * inv));
  if (lse && ch == 0 && piece == 0) lse[(long long)t * kH + h] = L > 0.f ? M + logf(L) : -INFINITY;
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(ptr);
  }
  return fn;
}

// q viewed as [rows][576] bf16, boxes of 64 values x 128 rows, 128-byte swizzle
bool make_q_map(CUtensorMap *m, const void *q, unsigned long long rows) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDk, rows};
  cuuint64_t strides[1] = {(cuuint64_t)kRowBytes};
  cuuint32_t box[2] = {64, (cuuint32_t)kH};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(q), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The latent cache viewed as [rows][576] bf16 for four-row gathers: boxes of 64
// values x 1 row, 128-byte swizzle (the score and value tiles' layout).
bool make_kv_gather_map(CUtensorMap *m, const void *kv, unsigned long long rows) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDk, rows};
  cuuint64_t strides[1] = {(cuuint64_t)kRowBytes};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(kv), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Rows of the latent cache under layout L (paged pool or [B][n_max]); 0 when the
// count does not fit a gather coordinate.
int kv_rows_of(const Layout &L) {
  const long long rows = L.page_size ? (long long)L.num_pages * L.page_size : (long long)L.batch * L.n_max;
  return rows > 0 && rows < 0x7FFFFFFFll ? (int)rows : 0;
}

size_t part_bytes_per_row(int splits) {
  return (size_t)splits * kH * (kDv * sizeof(__half) + sizeof(float2));
}

}  // namespace

bool make_q576_map(CUtensorMap *m, const void *q, unsigned long long rows) { return make_q_map(m, q, rows); }

bool make_bf16_rows_map(CUtensorMap *m, const void *base, unsigned long long rows, unsigned width) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)width, rows};
  cuuint64_t strides[1] = {(cuuint64_t)width * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kH};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

AttnPlan attn_bf16_plan(int T, int k, int num_sms) {
  (void)T;
  (void)num_sms;
  AttnPlan pl;
  pl.keys_per_split = k >= kMaxKeys ? kMaxKeys : ((k + 63) / 64) * 64;
  pl.splits = (k + pl.keys_per_split - 1) / pl.keys_per_split;
  return pl;
}

size_t attn_bf16_workspace(int T, int k, int num_sms) {
  const AttnPlan pl = attn_bf16_plan(T, k, num_sms);
  const int rows = T < kRowsPerLaunch ? T : kRowsPerLaunch;
  return (size_t)rows * part_bytes_per_row(pl.splits);
}

cudaError_t launch_attn_bf16(const void *q, const void *kv, int T, float scale, const int *idx, int k,
                             const Layout &L, void *out, float *lse, void *ws, size_t ws_bytes, const ErrCtx &e,
                             int num_sms, cudaStream_t stream) {
  const AttnPlan pl = attn_bf16_plan(T, k, num_sms);
  const int rows_max = T < kRowsPerLaunch ? T : kRowsPerLaunch;
  if (ws_bytes < (size_t)rows_max * part_bytes_per_row(pl.splits)) return cudaErrorInvalidValue;
  cudaError_t err = cudaFuncSetAttribute(attn_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (err != cudaSuccess) return err;
  Params p;
  p.kv_rows = kv_rows_of(L);
  CUtensorMap tkv;
  if (p.kv_rows == 0 || !make_kv_gather_map(&tkv, kv, (unsigned long long)p.kv_rows)) return cudaErrorInvalidValue;
  p.k = k;
  p.splits = pl.splits;
  p.keys_per_split = pl.keys_per_split;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o_part = static_cast<__half *>(ws);
  p.ml_part = reinterpret_cast<float2 *>(static_cast<char *>(ws) +
                                         (size_t)rows_max * pl.splits * kH * kDv * sizeof(__half));
  p.e = e;
  for (int r0 = 0; r0 < T; r0 += kRowsPerLaunch) {
    const int nr = T - r0 < kRowsPerLaunch ? T - r0 : kRowsPerLaunch;
    CUtensorMap tq;
    const char *qc = static_cast<const char *>(q) + (size_t)r0 * kH * kRowBytes;
    if (!make_q_map(&tq, qc, (unsigned long long)nr * kH)) return cudaErrorInvalidValue;
    p.idx = idx + (size_t)r0 * k;
    p.L = L;
    p.L.row0 = L.row0 + r0;
    err = launch_kernel(attn_bf16_kernel, dim3(nr * pl.splits), dim3(kThreads), kSmem, stream, 0, tq, tkv, p);
    if (err != cudaSuccess) return err;
    err = launch_kernel(attn_combine_kernel, dim3(nr, (kDv / 64) * kCombPer), dim3(kCombThreads), 0, stream, 0,
                        static_cast<const __half *>(p.o_part), static_cast<const float2 *>(p.ml_part), pl.splits,
                        static_cast<__nv_bfloat16 *>(out) + (size_t)r0 * kH * kDv,
                        lse ? lse + (size_t)r0 * kH : nullptr);
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}


// ------------------------------------------------------------------ built-in scratch
// For callers that may not allocate device memory: the split partials live in
// this file-scope array instead of a caller workspace. Host code must not pass
// the symbol itself to a kernel (on the host it names a shadow variable, not
// device memory): its device address is looked up once per device below.
namespace {
constexpr size_t kScratchBytes = size_t(40) << 20;  // 40 MiB, held by every GPU that loads the library
static __device__ __align__(256) unsigned char g_attn_scratch[kScratchBytes];

constexpr int kScratchDevices = 64;
void *g_scratch_addr[kScratchDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (looked up on the
// first call per device, with that device current).
cudaError_t scratch_address(void **out) {
  int dev = -1;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kScratchDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void *ptr = nullptr;
    err = cudaGetSymbolAddress(&ptr, g_attn_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}
}  // namespace

size_t attn_bf16_scratch_limit() { return kScratchBytes; }

cudaError_t attn_bf16_scratch_setup() {
  void *scratch = nullptr;
  return scratch_address(&scratch);
}

size_t attn_bf16_scratch_bytes(int T, int k) {
  const AttnPlan pl = attn_bf16_plan(T, k, 0);
  return (size_t)T * part_bytes_per_row(pl.splits);
}

cudaError_t launch_attn_bf16_noalloc(const void *q, const void *kv, int T, float scale, const int *idx, int k,
                                     const Layout &L, void *out, float *lse, const ErrCtx &e, int num_sms,
                                     cudaStream_t stream) {
  (void)num_sms;
  const AttnPlan pl = attn_bf16_plan(T, k, num_sms);
  const size_t need = (size_t)T * part_bytes_per_row(pl.splits);
  if (need > kScratchBytes) return cudaErrorInvalidValue;
  void *scratch = nullptr;
  cudaError_t err = scratch_address(&scratch);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(attn_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (err != cudaSuccess) return err;
  CUtensorMap tq;
  if (!make_q_map(&tq, q, (unsigned long long)T * kH)) return cudaErrorInvalidValue;
  Params p;
  p.kv_rows = kv_rows_of(L);
  CUtensorMap tkv;
  if (p.kv_rows == 0 || !make_kv_gather_map(&tkv, kv, (unsigned long long)p.kv_rows)) return cudaErrorInvalidValue;
  p.idx = idx;
  p.k = k;
  p.splits = pl.splits;
  p.keys_per_split = pl.keys_per_split;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o_part = static_cast<__half *>(scratch);
  p.ml_part = reinterpret_cast<float2 *>(static_cast<char *>(scratch) +
                                         (size_t)T * pl.splits * kH * kDv * sizeof(__half));
  p.L = L;
  p.e = e;
  err = launch_kernel(attn_bf16_kernel, dim3(T * pl.splits), dim3(kThreads), kSmem, stream, 0, tq, tkv, p);
  if (err != cudaSuccess) return err;
  return launch_kernel(attn_combine_kernel, dim3(T, (kDv / 64) * kCombPer), dim3(kCombThreads), 0, stream, 0,
                       static_cast<const __half *>(p.o_part), static_cast<const float2 *>(p.ml_part), pl.splits,
                       static_cast<__nv_bfloat16 *>(out), lse);
}

}  // namespace dsa
