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
//   2. Eight warps (one head row per thread, two per TMEM lane quadrant) read S
//      from TMEM, take the row max and write P = exp(scale (S - max)) as bf16 back
//      into TMEM, where the value MMAs take it as their A operand.
//   3. O[128, 512] = P[128, n] . V[n, 512], 128 values (two 64-dim chunks, one
//      MN-major B operand from shared memory) at a time. The key tiles of chunks 6
//      and 7 are still in the ring when the score MMAs end and serve as the values
//      384..511 directly; chunks 0+1 are gathered during the score phase into the
//      shared memory P does not need, chunks 4+5 into the ring's freed query slots,
//      chunks 2+3 into the space of 6+7 once their MMAs are done.
//   4. O, normalised by the split's own sum, leaves in three parts as each is
//      complete, each staged as fp16 in freed shared memory and written with bulk
//      stores: values 256..511 and then 0..127 while later MMAs run, 128..255 last.
//      The row max and sum go beside it; a second kernel merges the splits of each
//      row with log-sum-exp weights.
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
constexpr int kRing = kStages * kStage;        // 144 KiB
constexpr int kHalfTile = 128 * 128;           // 128 rows of one 64-dim chunk, 16 KiB
constexpr int kVSlot = 2 * kKTile;             // 64 KiB: value chunks 0 and 1 (the space P would take)
constexpr uint32_t kPCol = 384;                // TMEM columns of P: 128 (two bf16 per column)
constexpr int kProducerWarps = 4;              // warps 0-3
constexpr int kMmaWarp = 4;
constexpr int kSmWarp0 = 5, kSmWarps = 8;      // softmax/output warps: two per TMEM lane quadrant
constexpr int kThreads = 32 * (4 + 1 + kSmWarps);
static_assert(kThreads >= kMaxKeys, "one selection entry per thread");
constexpr int kSmem = 1024 + kRing + kVSlot + kMaxKeys * 4 + 256 + 1024;
constexpr int kRowsPerLaunch = 74;             // rows per launch: 74 x 8 splits = four waves of 148 CTAs, and
                                               // the launch's fp16 partials (74 MB) stay in L2 for the merge
constexpr int kSlice = kH * 128;               // partial output of 64 values of all heads (fp16)
static_assert(kChunks == 9 && kStages == 3, "the value phase reads chunks 6 and 7 from ring stages 0 and 1");

// Value phase: the pairs of 64-dim chunks in MMA order, where each pair's rows
// 0..127 and 128..255 lie in shared memory (byte offsets from the ring's start;
// the second chunk of a pair sits `lbo` bytes after the first, the operand's
// stride between 64-value groups), and the TMEM column its 128 outputs go to.
//   pair 0, chunks 6+7: the key tiles of ring stages 0 and 1, left in place;
//   pair 1, chunks 4+5: the query slots of stages 0 and 1 and stage 2's first
//                       32 KiB, free once the score MMAs are done;
//   pair 2, chunks 0+1: the slot after the ring, gathered during the score phase;
//   pair 3, chunks 2+3: pair 0's space once pair 0's MMAs are done.
// TMEM: S in columns 0..255 until P is written, P in 384..511; pair 0's outputs in
// 256..383, pair 1's in 0..127, pair 2's in 128..255, pair 3's in 256..383 once
// pair 0's have been read out.
struct VPair {
  int chunk0;      // first chunk of the pair (values 64 * chunk0 ..)
  int off0, off1;  // byte offset of the first chunk's rows 0..127 / 128..255
  int lbo0, lbo1;  // byte distance to the second chunk's rows, per row half
  uint32_t dcol;   // TMEM column of the pair's first output value
  __device__ __forceinline__ int off(int h) const { return h ? off1 : off0; }
  __device__ __forceinline__ int lbo(int h) const { return h ? lbo1 : lbo0; }
};
__device__ __forceinline__ VPair vpair(int i) {
  VPair v;
  if (i == 0 || i == 3) {  // key tiles of stages 0 and 1: chunk at +16 KiB, rows 128.. at +16 KiB more
    v.chunk0 = i == 0 ? 6 : 2;
    v.off0 = kQTile;
    v.off1 = kQTile + kHalfTile;
    v.lbo0 = v.lbo1 = kStage;
    v.dcol = 256;
  } else if (i == 1) {     // the query slots of stages 0 and 1, and stage 2's first 32 KiB
    v.chunk0 = 4;
    v.off0 = 0;
    v.off1 = 2 * kStage;
    v.lbo0 = kStage;
    v.lbo1 = kHalfTile;
    v.dcol = 0;
  } else {                 // the slot after the ring: chunk 0 then chunk 1, 32 KiB each
    v.chunk0 = 0;
    v.off0 = kRing;
    v.off1 = kRing + kHalfTile;
    v.lbo0 = v.lbo1 = kKTile;
    v.dcol = 128;
  }
  return v;
}
// TMEM column holding output value d (0..511)
__device__ __forceinline__ uint32_t out_col(int d) {
  const int i = d >= 384 ? 0 : d >= 256 ? 1 : d < 128 ? 2 : 3;
  const VPair v = vpair(i);
  return v.dcol + (uint32_t)(d - 64 * v.chunk0);
}
// Staging of 64-value output chunk c (fp16 [128 heads][64], 16 KiB) before its bulk
// store: values 256..511 in pair 1's space (free once its MMAs are done), values
// 0..255 in the slot after the ring, pair 2's space (free once pair 2's MMAs are
// done; values 0..127 are staged then, 128..255 after the last MMA).
__device__ __forceinline__ int stage_off(int c) {
  if (c < 4) return kRing + c * kSlice;
  const int i = c - 4;  // query slot of stage 0, of stage 1, then stage 2's first two 16 KiB
  return i < 2 ? i * kStage : 2 * kStage + (i - 2) * kSlice;
}

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
  unsigned char *ring = base;  // score ring, then value tiles and output staging; the value slot follows it
  int *rows = reinterpret_cast<int *>(base + kRing + kVSlot);  // gather row of each selected entry
  uint64_t *bars = reinterpret_cast<uint64_t *>(rows + kMaxKeys);
  uint64_t *full = bars, *empty = bars + kStages;
  uint64_t *vfull = bars + 2 * kStages;  // value pairs 1..3 gathered
  uint64_t *vdone = vfull + 4;           // value pair 0 consumed (its space is free)
  uint64_t *s_full = vdone + 1, *p_full = s_full + 1;
  uint64_t *o_done = p_full + 1;         // outputs complete: values 256..511, 0..127, 128..255
  uint64_t *o_lo = o_done + 2;           // (the last one: every MMA of this CTA complete)
  uint64_t *hi_read = o_lo + 1;          // the outputs of values 256..511 are out of TMEM
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(hi_read + 1);
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

  // ---- barriers and TMEM (they do not depend on the selection, so they overlap
  // its loads), then the selected rows of this split (-1 entries are padding,
  // anywhere in the list)
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, kProducerWarps);
      mbar_init(empty + s, 1);
    }
    for (int j = 1; j < 4; ++j) mbar_init(vfull + j, kProducerWarps);
    mbar_init(vdone, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, kSmWarps);
    for (int j = 0; j < 3; ++j) mbar_init(o_done + j, 1);
    mbar_init(hi_read, kSmWarps);
    fence_mbar_init();
    s_nvalid = 0;
  }
  if (threadIdx.x < kMaxKeys / 32) s_valid[threadIdx.x] = 0;
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  const RowPos rp = row_position(p.L, t);
  const int i = threadIdx.x;  // entry i of the split's selection (kThreads >= kMaxKeys)
  const int sel = i < nk && i < kMaxKeys ? __ldg(p.idx + (long long)t * p.k + k0 + i) : -1;
  tc_fence_before();
  __syncthreads();  // s_nvalid, s_valid and the barriers are initialised
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (i < kMaxKeys) {
    long long r = -1;
    if (i < nk) {
      if (sel >= 0 && sel <= rp.pos && rp.len <= cache_capacity(p.L)) {
        r = key_row(p.L, rp.b, sel, p.e, 0x500);
      } else if (sel != -1) {
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
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
    return;
  }
  const int n = ((nvalid + 63) / 64) * 64;  // MMA N of the score tile, K of the value MMAs

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
    // value pairs: 2 now (its slot is free from the start), 1 once every score MMA has
    // consumed the ring, 3 once pair 0's MMAs have consumed its space
    for (int k = 0; k < 3 && ok; ++k) {
      const int i = k == 0 ? 2 : k == 1 ? 1 : 3;
      if (i == 1) ok = mbar_wait(s_full, 0, p.e, 0x511);
      if (i == 3) ok = mbar_wait(vdone, 0, p.e, 0x512);
      if (!ok) break;
      const VPair v = vpair(i);
      // 2 chunks x n/4 row groups; thread q = 4 * lane + warp takes chunk q >> 6, group q & 63
      const int q = 4 * lane + warp, j = q >> 6, g = q & 63;
      const bool mine = g < n / 4;
      const unsigned cnt = __popc(__ballot_sync(0xFFFFFFFFu, mine));
      if (lane == 0) mbar_expect_tx(vfull + i, cnt * 512);
      __syncwarp();
      if (mine) {
        const int h = g >> 5;  // row half
        unsigned char *dst = ring + v.off(h) + j * v.lbo(h) + (g & 31) * 512;
        tma_gather4(dst, &tm_kv, vfull + i, (v.chunk0 + j) * 64, rows[4 * g], rows[4 * g + 1], rows[4 * g + 2],
                    rows[4 * g + 3]);
      }
    }
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = instr_desc(1, 1, 0, 0, 128, (uint32_t)n);
      const uint32_t r0 = smem_u32(ring);
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
      // O[:, 64 c0 .. 64 c0 + 127] = P . V over n rows in K steps of 16 rows (8 TMEM columns of P each)
      const uint32_t idesc_pv = instr_desc(1, 1, 0, 1, 128, 128);  // B MN-major, N = 128
      for (int i = 0; i < 4 && ok; ++i) {
        if (i > 0) {
          ok = mbar_wait(vfull + i, 0, p.e, 0x522);
          if (ok && i == 3) ok = mbar_wait(hi_read, 0, p.e, 0x523);  // pair 3 reuses pair 0's columns
          if (!ok) break;
          tc_fence_after();
        }
        const VPair v = vpair(i);
        for (int ks = 0; ks < n / 16; ++ks) {
          const int h = ks >> 3;  // row half
          const uint64_t bd = smem_desc(r0 + v.off(h) + (ks & 7) * 2048, (uint32_t)v.lbo(h), 1024, SW_128B);
          umma_f16_ts(tmem + v.dcol, tmem + kPCol + ks * 8, bd, idesc_pv, ks != 0);
        }
        if (i == 0) umma_commit(vdone);
        if (i == 1) umma_commit(o_done);      // values 256..511 complete
        if (i == 2) umma_commit(o_done + 1);  // values 0..127 complete
      }
      umma_commit(o_lo);  // every MMA of this CTA complete
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
          if (vm == 0xFFFFFFFFu) {  // every entry of the chunk is a real row: a plain tree
            float t8[8];
#pragma unroll
            for (int y = 0; y < 8; ++y)
              t8[y] = fmaxf(fmaxf(__uint_as_float(v[u][4 * y]), __uint_as_float(v[u][4 * y + 1])),
                            fmaxf(__uint_as_float(v[u][4 * y + 2]), __uint_as_float(v[u][4 * y + 3])));
            m = fmaxf(m, fmaxf(fmaxf(fmaxf(t8[0], t8[1]), fmaxf(t8[2], t8[3])),
                               fmaxf(fmaxf(t8[4], t8[5]), fmaxf(t8[6], t8[7]))));
          } else {
#pragma unroll
            for (int x = 0; x < 32; ++x)
              if ((vm >> x) & 1u) m = fmaxf(m, __uint_as_float(v[u][x]));
          }
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
        // keys j*32 .. j*32+31: 16 TMEM columns of P, two keys per column
        tmem_st16(trow + kPCol + j * 16, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    s_part[half][h] = l;
    softmax_bar();
    l = s_part[0][h] + s_part[1][h];
    // this warp's 256 output values in three parts, normalised by the split's own sum
    // (a convex combination of value rows, so fp16 keeps ~1e-3 absolute accuracy):
    // staged in the workspace's layout (64-value chunks of [128 heads][64], the
    // 16-byte pieces of a head swizzled by the head's low three bits), then bulk stores
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    char *ob = reinterpret_cast<char *>(p.o_part + part * (long long)(kDv * kH));
    for (int pt = 0; pt < 3; ++pt) {  // values 256..511, then 0..127, then 128..255
      const int lo = pt == 0 ? 256 : pt == 1 ? 0 : 128, width = pt == 0 ? 256 : 128;
      if (ok) ok = mbar_wait(pt == 2 ? o_lo : o_done + pt, 0, p.e, 0x531);
      if (ok) {
        tc_fence_after();
        const int d0 = lo + half * (width / 2);  // this warp's values
        for (int d = d0; d < d0 + width / 2; d += 64) {
          uint32_t v[2][32];
          tmem_ld32(trow + out_col(d), v[0]);
          tmem_ld32(trow + out_col(d + 32), v[1]);
          tmem_ld_wait(v[0]);
          tmem_ld_wait(v[1]);
          unsigned char *cb = ring + stage_off(d >> 6) + h * 128;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
#pragma unroll
            for (int pc = 0; pc < 4; ++pc) {
              uint32_t w[4];
#pragma unroll
              for (int y = 0; y < 4; ++y)
                w[y] = pack_half(__uint_as_float(v[u][pc * 8 + 2 * y]) * inv_l,
                                 __uint_as_float(v[u][pc * 8 + 2 * y + 1]) * inv_l);
              const int piece = u * 4 + pc;
              *reinterpret_cast<uint4 *>(cb + ((piece ^ (h & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
        fence_proxy_async_smem();
      }
      if (pt == 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(hi_read);  // pair 3 may overwrite these TMEM columns
      }
      softmax_bar();  // the part is staged
      if (ok && sw == 0 && lane == 0) {
        for (int c = lo / 64; c < (lo + width) / 64; ++c) bulk_store(ob + c * kSlice, ring + stage_off(c), kSlice);
        bulk_commit();
      }
    }
    if (sw == 0 && lane == 0) bulk_wait_read_all();  // the staged tiles are read before this CTA ends
    if (half == 0) p.ml_part[part * kH + h] = ok ? make_float2(m * p.scale, l) : make_float2(-INFINITY, 0.f);
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
    // all MMAs have completed once o_lo fired; if a wait gave up, wait here (bounded)
    if (lane == 0) mbar_wait(o_lo, 0, p.e, 0x540);
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
