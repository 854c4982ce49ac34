// Fine-grained token selection: per query row, the k best indexer scores over
// the row's causal prefix (jdon.com "DeepSeek-V3.2-Exp", sparse-training and
// selection paragraphs: K = 2048 tokens kept per query; openi.cn "DeepSeek-V3.2",
// token-selection item).
//
// One thread-block cluster of C CTAs per row. Each CTA holds a contiguous slice
// of the row in shared memory as order-preserving 32-bit keys and builds the
// histogram of their top 12 bits while loading. Each CTA sums one slice of the
// bins over the cluster and writes the totals into every peer, so all CTAs find
// the bin holding the k-th best key. Keys in that bin are the only candidates
// whose fate is open (about 1% of a long row): every CTA gathers the whole
// row's candidates and finishes the radix select on them locally (bits 19..10,
// then 9..0). The scan that finds the candidates also lists, per warp and in
// position order, every key at or above the candidates' bin; the selected ones
// among them (keys above the threshold plus the lowest-position keys equal to it)
// are written in ascending order with warp ballots.
// When the candidates do not fit (very flat score rows) or many keys tie at the
// threshold, the cluster falls back to full radix passes over all keys. The row
// is read from memory exactly once.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins1 = 4096, kBins2 = 1024, kBins3 = 1024;  // bits 31..20, 19..10, 9..0

// Monotone map float -> uint32: larger float, larger key; -0 and +0 share a key;
// every NaN maps below -inf.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kW1 = kBins1 / kThreads, kW2 = kBins2 / kThreads;  // bins per thread in the scans
constexpr int kCandCap = 1024;  // candidates per CTA
constexpr int kAllCap = 2048;   // candidates per row
constexpr int kLaneCand = kAllCap / kThreads;  // per thread while scanning
constexpr int kOvfCap = 256;                    // candidates beyond a thread's slots, per CTA
constexpr int kTieCap = 64;     // keys equal to the threshold resolved on the fast path
constexpr int kWList = (kBins1 - kBins2) * 2 / kWarps;  // listed keys per warp (in hist1 past bin 1023)

struct Shared {
  unsigned hist1[kBins1];  // this CTA's histogram of bits 31..20, then the cluster totals; later
                           // the candidates' histograms
  uint2 cand[kCandCap];    // this CTA's candidates: (key, position in the row)
  uint2 ovf[kOvfCap];      // candidates of threads whose slots are full
  union {
    uint2 allc[kAllCap];   // the whole row's candidates (while scanning: per-thread candidate slots)
    struct {
      unsigned hist2[kBins2], hist3[kBins3];
    } slow;
  } u;
  unsigned wsum[kWarps];
  unsigned wsum2[kWarps];
  unsigned wgt[kWarps];    // per warp segment: keys above the first-pass bin
  unsigned wsel[kWarps];   // per warp segment: selected candidates
  unsigned wn[kWarps];     // per warp segment: keys at or above the candidates' bin
  uint2 pub;               // (keys above the first-pass bin, candidates) of this CTA, read by the peers
  unsigned cta_cnt[2];     // (greater, equal) counts of this CTA, read by the peers (fallback)
  unsigned sel_before, ntie, novf;
  int tie_pos[kTieCap];
  int tie_cut;
  unsigned sel_bin, sel_krem;
  unsigned out_base, eq_take;
};

// Each thread holds the cluster-wide counts of W consecutive bins
// [tid*W, tid*W + W). Finds, scanning from the highest bin down, the bin that
// holds the krem-th largest key; stores it and the rank left inside it.
template <int W>
__device__ __forceinline__ void find_bin(const unsigned (&v)[W], unsigned krem, Shared &sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned s = 0;
#pragma unroll
  for (int i = 0; i < W; ++i) s += v[i];
  unsigned incl = s;  // suffix sum over lanes >= lane
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned o = __shfl_down_sync(0xFFFFFFFFu, incl, off);
    if (lane + off < 32) incl += o;
  }
  if (lane == 0) sm.wsum[warp] = incl;
  __syncthreads();
  unsigned above = incl - s;
#pragma unroll
  for (int w = 0; w < kWarps; ++w)
    if (w > warp) above += sm.wsum[w];
  if (above < krem && krem <= above + s) {
    unsigned c = above;
#pragma unroll
    for (int i = W - 1; i >= 0; --i) {
      if (c + v[i] >= krem) {
        sm.sel_bin = (unsigned)(tid * W + i);
        sm.sel_krem = krem - c;
        break;
      }
      c += v[i];
    }
  }
  __syncthreads();
}

// Sum over the cluster of W (1, 2 or 4) consecutive bins per thread (all peers read at once).
template <int C, int W>
__device__ __forceinline__ void cluster_counts(cg::cluster_group &cluster, unsigned *h, unsigned (&v)[W]) {
  const int tid = threadIdx.x;
  unsigned peer[C][W];
#pragma unroll
  for (int r = 0; r < C; ++r) {
    const unsigned *ph = cluster.map_shared_rank(h, r) + tid * W;
    if (W == 4) {
      const uint4 q = *reinterpret_cast<const uint4 *>(ph);
      peer[r][0] = q.x;
      peer[r][1 % W] = q.y;
      peer[r][2 % W] = q.z;
      peer[r][3 % W] = q.w;
    } else if (W == 2) {
      const uint2 q = *reinterpret_cast<const uint2 *>(ph);
      peer[r][0] = q.x;
      peer[r][1 % W] = q.y;
    } else {
      peer[r][0] = *ph;
    }
  }
#pragma unroll
  for (int i = 0; i < W; ++i) {
    unsigned a = 0;
#pragma unroll
    for (int r = 0; r < C; ++r) a += peer[r][i];
    v[i] = a;
  }
}

// Exclusive prefix over the block of a per-thread pair (a, b); returns the
// block totals through the references.
__device__ __forceinline__ void block_scan2(unsigned &a, unsigned &b, unsigned &tot_a, unsigned &tot_b,
                                            Shared &sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned ia = a, ib = b;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned oa = __shfl_up_sync(0xFFFFFFFFu, ia, off);
    const unsigned ob = __shfl_up_sync(0xFFFFFFFFu, ib, off);
    if (lane >= off) {
      ia += oa;
      ib += ob;
    }
  }
  if (lane == 31) {
    sm.wsum[warp] = ia;
    sm.wsum2[warp] = ib;
  }
  __syncthreads();
  unsigned pa = 0, pb = 0, ta = 0, tb = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const unsigned x = sm.wsum[w], y = sm.wsum2[w];
    if (w < warp) {
      pa += x;
      pb += y;
    }
    ta += x;
    tb += y;
  }
  a = pa + ia - a;
  b = pb + ib - b;
  tot_a = ta;
  tot_b = tb;
  __syncthreads();
}

template <int C>
__global__ void __launch_bounds__(kThreads) topk_kernel(const float *__restrict__ scores, long long ld, int k,
                                                        Layout L, int cap, int *__restrict__ idx, ErrCtx e) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Shared &sm = *reinterpret_cast<Shared *>(smem_raw);
  uint32_t *keys = reinterpret_cast<uint32_t *>(smem_raw + ((sizeof(Shared) + 15) & ~size_t(15)));

  pdl_prologue();
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int t = blockIdx.x / C;
  const int tid = threadIdx.x;

  const RowPos rp = row_position(L, t);
  long long n = (long long)rp.pos + 1;
  int *out = idx + (long long)t * k;
  if (rp.pos < 0 || n > ld || n > (long long)C * cap) {
    if (tid == 0 && rank == 0) raise_error(e, DEV_BOUNDS, 0x100);
    n = n < 0 ? 0 : n;
    n = n > ld ? ld : n;
    n = n > (long long)C * cap ? (long long)C * cap : n;
  }

  if (n <= k) {  // everything before the row's position is selected
    for (long long i = (long long)rank * kThreads + tid; i < k; i += (long long)C * kThreads)
      out[i] = i < n ? (int)i : -1;
    return;  // no distributed shared memory was touched
  }

  for (int i = tid; i < kBins1; i += kThreads) sm.hist1[i] = 0;
  if (tid == 0) sm.novf = 0;
  __syncthreads();

  // ---- this CTA's slice as keys in shared memory; histogram of bits 31..20
  const int chunk = (int)((((n + C - 1) / C) + 31) / 32 * 32);
  const long long lo = (long long)rank * chunk;
  const int cnt = (int)max(0LL, min(n, lo + chunk) - lo);
  {
    const float *row = scores + (long long)t * ld + lo;
    const int n4 = cnt >> 2;
    const float4 *r4 = reinterpret_cast<const float4 *>(row);
    constexpr int U = 4;  // float4 loads in flight per thread
    for (int base = 0; base < n4; base += U * kThreads) {
      float4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + u * kThreads + tid;
        if (i < n4) v[u] = __ldcs(r4 + i);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + u * kThreads + tid;
        if (i < n4) {
          const uint4 kk = make_uint4(order_key(v[u].x), order_key(v[u].y), order_key(v[u].z), order_key(v[u].w));
          reinterpret_cast<uint4 *>(keys)[i] = kk;
          atomicAdd(sm.hist1 + (kk.x >> 20), 1u);
          atomicAdd(sm.hist1 + (kk.y >> 20), 1u);
          atomicAdd(sm.hist1 + (kk.z >> 20), 1u);
          atomicAdd(sm.hist1 + (kk.w >> 20), 1u);
        }
      }
    }
    const int i = (n4 << 2) + tid;  // 0..3 trailing keys
    if (i < cnt) {
      const uint32_t kx = order_key(__ldcs(row + i));
      keys[i] = kx;
      atomicAdd(sm.hist1 + (kx >> 20), 1u);
    }
  }

  // ---- pass 1 (bits 31..20): this CTA sums bins [rank*S, rank*S + S) over the
  // cluster and writes the totals back into every CTA's histogram (only this CTA
  // touches those bins anywhere in the cluster)
  cluster.sync();
  {
    constexpr int S = kBins1 / C;
    for (int b = tid; b < S; b += kThreads) {
      const int bin = rank * S + b;
      unsigned part[C];
#pragma unroll
      for (int r = 0; r < C; ++r) part[r] = *cluster.map_shared_rank(sm.hist1 + bin, r);
      unsigned tot = 0;
#pragma unroll
      for (int r = 0; r < C; ++r) tot += part[r];
#pragma unroll
      for (int r = 0; r < C; ++r) *cluster.map_shared_rank(sm.hist1 + bin, r) = tot;
    }
  }
  cluster.sync();
  uint32_t b1;
  unsigned krem1;
  {
    unsigned v[kW1];
#pragma unroll
    for (int i = 0; i < kW1; ++i) v[i] = sm.hist1[tid * kW1 + i];
    find_bin<kW1>(v, (unsigned)k, sm);
    b1 = sm.sel_bin;
    krem1 = sm.sel_krem;
  }

  // ---- one scan of the slice: keys above bin b1 per warp segment, keys in it as
  // candidates. Warp w owns keys [w*seg, w*seg + seg); each lane reads 4 keys at a time
  // and keeps its candidates in slots of its own.
  const uint4 *keys4 = reinterpret_cast<const uint4 *>(keys);
  const int lane = tid & 31, warp = tid >> 5;
  const int seg = ((cnt + kWarps - 1) / kWarps + 127) / 128 * 128;
  const int s0 = min(cnt, warp * seg), s1 = min(cnt, s0 + seg);
  // hist1 past its first kBins2 bins is free from here on: the per-warp key lists
  uint16_t *wlist = reinterpret_cast<uint16_t *>(sm.hist1 + kBins2) + warp * kWList;
  {
    const uint32_t above = (b1 << 20) | 0xFFFFFu;  // keys greater than this lie above bin b1
    const uint32_t lowest = b1 << 20;              // keys at or above this: bin b1 or above
    const unsigned lt = (1u << lane) - 1u;
    unsigned ngt = 0, nc = 0, wn = 0;
    uint2 *mine = sm.u.allc + tid * kLaneCand;
    for (int i = s0 + 4 * lane; i - 4 * lane < s1; i += 128) {  // the same trip count in every lane
      const uint4 q = i < s1 ? keys4[i >> 2] : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t kk[4] = {q.x, q.y, q.z, q.w};
      bool ge[4];
      unsigned m[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool ok = i + j < s1;
        ge[j] = ok && kk[j] >= lowest;
        m[j] = __ballot_sync(0xFFFFFFFFu, ge[j]);
        ngt += ok && kk[j] > above;
        if (ok && (kk[j] >> 20) == b1) {
          const uint2 c = make_uint2(kk[j], (unsigned)(lo + i + j));
          if (nc < (unsigned)kLaneCand) {
            mine[nc++] = c;
          } else {
            const unsigned at = atomicAdd(&sm.novf, 1u);
            if (at < (unsigned)kOvfCap) sm.ovf[at] = c;
          }
        }
      }
      const unsigned tot = __popc(m[0]) + __popc(m[1]) + __popc(m[2]) + __popc(m[3]);
      if (tot == 0u) continue;
      // listed in position order: lane l's keys 4l .. 4l+3 after those of the lanes below it
      unsigned at = wn + __popc(m[0] & lt) + __popc(m[1] & lt) + __popc(m[2] & lt) + __popc(m[3] & lt);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (ge[j]) {
          if (at < (unsigned)kWList) wlist[at] = (uint16_t)(i + j - s0);
          ++at;
        }
      }
      wn += tot;
    }
    if (lane == 0) sm.wn[warp] = wn;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ngt += __shfl_xor_sync(0xFFFFFFFFu, ngt, off);
    if (lane == 0) sm.wgt[warp] = ngt;
    // compact the slots into this CTA's candidate list (read by the peers)
    unsigned off = nc, dummy = 0, tot, tot_dummy;
    block_scan2(off, dummy, tot, tot_dummy, sm);  // off: slot candidates of the threads before this one
    const unsigned novf = sm.novf;
    const bool over = novf > (unsigned)kOvfCap;
    tot += novf;
    if (!over && tot <= (unsigned)kCandCap) {
      for (unsigned j = 0; j < nc; ++j) sm.cand[off + j] = mine[j];
      for (unsigned j = tid; j < novf; j += kThreads) sm.cand[tot - novf + j] = sm.ovf[j];
    }
    if (tid == 0) {
      unsigned g = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) g += sm.wgt[w];
      // an overflowing list is published as too many candidates (the fallback path)
      sm.pub = make_uint2(g, over ? (unsigned)kCandCap + 1u : tot);
    }
  }
  cluster.sync();

  // ---- gather the row's candidates (every CTA the same list, in rank order)
  unsigned gt_before = 0, ncand_all = 0, cand_off[C];
  bool slow = false;
#pragma unroll
  for (int r = 0; r < C; ++r) {
    const uint2 pr = *cluster.map_shared_rank(&sm.pub, r);
    if (r < rank) gt_before += pr.x;
    cand_off[r] = ncand_all;
    ncand_all += pr.y;
    slow |= pr.y > (unsigned)kCandCap;
  }
  slow |= ncand_all > (unsigned)kAllCap;
  if (!slow) {
    // one pass over the concatenated lists: every peer's loads are in flight together
    for (unsigned f = tid; f < ncand_all; f += kThreads) {
      int r = 0;
      unsigned base = 0;
#pragma unroll
      for (int q = 1; q < C; ++q)
        if (f >= cand_off[q]) {
          r = q;
          base = cand_off[q];
        }
      sm.u.allc[f] = cluster.map_shared_rank(sm.cand, r)[f - base];
    }
  }
  cluster.sync();  // no CTA reads a peer's shared memory after this point on the fast path

  uint32_t thr = 0;
  if (!slow) {
    // ---- radix select among the candidates: bits 19..10, then 9..0
    const unsigned nc = ncand_all;
    for (int i = tid; i < kBins2; i += kThreads) sm.hist1[i] = 0;
    __syncthreads();
    for (unsigned j = tid; j < nc; j += kThreads) atomicAdd(sm.hist1 + ((sm.u.allc[j].x >> 10) & 1023u), 1u);
    __syncthreads();
    unsigned b2, krem2, b3, krem3;
    {
      unsigned v[kW2];
#pragma unroll
      for (int i = 0; i < kW2; ++i) v[i] = sm.hist1[tid * kW2 + i];
      find_bin<kW2>(v, krem1, sm);
      b2 = sm.sel_bin;
      krem2 = sm.sel_krem;
    }
    for (int i = tid; i < kBins3; i += kThreads) sm.hist1[i] = 0;
    if (tid == 0) {
      sm.ntie = 0;
      sm.sel_before = 0;
      sm.tie_cut = 0x7FFFFFFF;
    }
    if (tid < kWarps) sm.wsel[tid] = 0;
    __syncthreads();
    for (unsigned j = tid; j < nc; j += kThreads) {
      const uint32_t key = sm.u.allc[j].x;
      if (((key >> 10) & 1023u) == b2) atomicAdd(sm.hist1 + (key & 1023u), 1u);
    }
    __syncthreads();
    {
      unsigned v[kW2];
#pragma unroll
      for (int i = 0; i < kW2; ++i) v[i] = sm.hist1[tid * kW2 + i];
      find_bin<kW2>(v, krem2, sm);
      b3 = sm.sel_bin;
      krem3 = sm.sel_krem;
    }
    thr = (b1 << 20) | (b2 << 10) | b3;
    const unsigned ties = sm.hist1[b3];  // candidates equal to the threshold
    if (krem3 < ties) {
      // only the krem3 lowest positions among the ties are taken
      if (ties > (unsigned)kTieCap) {
        slow = true;  // the same decision in every CTA (same candidate list)
      } else {
        for (unsigned j = tid; j < nc; j += kThreads) {
          const uint2 c = sm.u.allc[j];
          if (c.x == thr) sm.tie_pos[atomicAdd(&sm.ntie, 1u)] = (int)c.y;
        }
        __syncthreads();
        if (warp == 0) {
#pragma unroll
          for (int q = 0; q < kTieCap / 32; ++q) {
            const unsigned a = lane + 32 * q;
            if (a < ties) {
              const int pa = sm.tie_pos[a];
              unsigned below = 0;
              for (unsigned b = 0; b < ties; ++b) below += sm.tie_pos[b] < pa;
              if (below == krem3 - 1) sm.tie_cut = pa;
            }
          }
        }
      }
    }
    __syncthreads();
  }

  if (!slow) {
    // ---- selected candidates: those of earlier CTAs, and per warp segment of this one
    const uint32_t tcut = (uint32_t)sm.tie_cut;
    unsigned sb = 0;  // selected candidates of earlier CTAs seen by this thread
    for (unsigned j = tid; j < ncand_all; j += kThreads) {
      const uint2 c = sm.u.allc[j];
      if (c.x > thr || (c.x == thr && c.y <= tcut)) {
        if ((long long)c.y < lo) {
          ++sb;
        } else if ((long long)c.y < lo + cnt) {
          atomicAdd(sm.wsel + (int)((long long)c.y - lo) / seg, 1u);
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sb += __shfl_xor_sync(0xFFFFFFFFu, sb, off);
    if (lane == 0 && sb) atomicAdd(&sm.sel_before, sb);
    __syncthreads();
    unsigned o = gt_before + sm.sel_before;
    for (int w = 0; w < warp; ++w) o += sm.wgt[w] + sm.wsel[w];
    // ---- emit this warp's selected keys in ascending position order, from its list
    // when every key at or above the candidates' bin fit into it
    const unsigned lt = (1u << lane) - 1u;
    const unsigned wn = sm.wn[warp];
    if (wn <= (unsigned)kWList) {
      for (unsigned b = 0; b < wn; b += 32) {
        const unsigned e = b + lane;
        bool sel = false;
        int r = 0;
        if (e < wn) {
          r = s0 + (int)wlist[e];
          const uint32_t key = keys[r];
          sel = key > thr || (key == thr && (uint32_t)(lo + r) <= tcut);
        }
        const unsigned m = __ballot_sync(0xFFFFFFFFu, sel);
        if (sel) {
          const unsigned at = o + __popc(m & lt);
          if (at < (unsigned)k) out[at] = (int)(lo + r);
        }
        o += __popc(m);
      }
    } else {
      for (int i = s0 + lane; i - lane < s1; i += 32) {
        const uint32_t key = i < s1 ? keys[i] : 0u;
        const bool sel = i < s1 && (key > thr || (key == thr && (uint32_t)(lo + i) <= tcut));
        const unsigned m = __ballot_sync(0xFFFFFFFFu, sel);
        if (sel) {
          const unsigned at = o + __popc(m & lt);
          if (at < (unsigned)k) out[at] = (int)(lo + i);
        }
        o += __popc(m);
      }
    }
    return;
  }

  // ================= fallback: full radix passes over every key of the slice
  for (int i = tid; i < kBins2; i += kThreads) sm.u.slow.hist2[i] = 0;
  for (int i = tid; i < kBins3; i += kThreads) sm.u.slow.hist3[i] = 0;
  __syncthreads();
  unsigned krem = krem1;
  uint32_t prefix = b1;
  // ---- pass 2: bits 19..10 among keys whose top 12 bits match
#pragma unroll 4
  for (int i = tid; i < cnt; i += kThreads) {
    const uint32_t key = keys[i];
    if ((key >> 20) == prefix) atomicAdd(sm.u.slow.hist2 + ((key >> 10) & 1023u), 1u);
  }
  cluster.sync();
  {
    unsigned v[kW2];
    cluster_counts<C, kW2>(cluster, sm.u.slow.hist2, v);
    find_bin<kW2>(v, krem, sm);
    prefix = (prefix << 10) | sm.sel_bin;  // top 22 bits
    krem = sm.sel_krem;
  }
  // ---- pass 3: bits 9..0 among keys whose top 22 bits match
#pragma unroll 4
  for (int i = tid; i < cnt; i += kThreads) {
    const uint32_t key = keys[i];
    if ((key >> 10) == prefix) atomicAdd(sm.u.slow.hist3 + (key & 1023u), 1u);
  }
  cluster.sync();
  {
    unsigned v[kW2];
    cluster_counts<C, kW2>(cluster, sm.u.slow.hist3, v);
    find_bin<kW2>(v, krem, sm);
    prefix = (prefix << 10) | sm.sel_bin;  // the threshold key
    krem = sm.sel_krem;                    // keys equal to it still to take
  }
  thr = prefix;

  // ---- each thread owns a contiguous run of the slice: counts, block scan, cluster scan
  const int run = (cnt + kThreads - 1) / kThreads;
  const int r0 = min(cnt, tid * run), r1 = min(cnt, r0 + run);
  unsigned gt = 0, eq = 0;
  for (int i = r0; i < r1; ++i) {
    const uint32_t key = keys[i];
    gt += key > thr;
    eq += key == thr;
  }
  unsigned cta_gt, cta_eq;
  block_scan2(gt, eq, cta_gt, cta_eq, sm);  // gt, eq now exclusive prefixes within the CTA
  if (tid == 0) {
    sm.cta_cnt[0] = cta_gt;
    sm.cta_cnt[1] = cta_eq;
  }
  cluster.sync();
  if (tid == 0) {
    unsigned pc[C][2];
#pragma unroll
    for (int r = 0; r < C; ++r) {
      const uint2 c2 = *reinterpret_cast<const uint2 *>(cluster.map_shared_rank(sm.cta_cnt, r));
      pc[r][0] = c2.x;
      pc[r][1] = c2.y;
    }
    unsigned gtb = 0, eqb = 0;
#pragma unroll
    for (int r = 0; r < C; ++r)
      if (r < rank) {
        gtb += pc[r][0];
        eqb += pc[r][1];
      }
    const unsigned taken_before = min(eqb, krem);
    sm.eq_take = min(cta_eq, krem - taken_before);
    sm.out_base = gtb + taken_before;
  }
  cluster.sync();  // peers are done reading this CTA's counts after this point

  // ---- emit this thread's selected positions in ascending order
  {
    const unsigned eq_take = sm.eq_take;
    unsigned tie = eq;                                  // ties before this thread's run
    unsigned o = sm.out_base + gt + min(eq, eq_take);   // selected before this thread's run
    for (int i = r0; i < r1; ++i) {
      const uint32_t key = keys[i];
      bool take = key > thr;
      if (key == thr) {
        take = tie < eq_take;
        ++tie;
      }
      if (take) {
        if (o < (unsigned)k) out[o] = (int)(lo + i);
        ++o;
      }
    }
  }
}

template <int C>
cudaError_t launch_c(const float *scores, long long ld, int T, int k, const Layout &L, int cap, int *idx,
                     const ErrCtx &e, cudaStream_t stream) {
  const size_t smem = topk_smem_bytes(cap);
  cudaError_t err = cudaFuncSetAttribute(topk_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  // all of L1 as shared memory, so that two CTAs of up to ~113 KB fit on one SM
  // (clusters of 8 then need only half a GPC each)
  err = cudaFuncSetAttribute(topk_kernel<C>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (err != cudaSuccess) return err;
  return launch_kernel(topk_kernel<C>, dim3((unsigned)T * C), dim3(kThreads), smem, stream, (unsigned)C, scores, ld, k, L,
                       cap, idx, e);
}

}  // namespace

size_t topk_smem_bytes(int cap) { return ((sizeof(Shared) + 15) & ~size_t(15)) + (size_t)cap * 4; }

cudaError_t launch_topk(const float *scores, long long ld, int T, int k, const Layout &L, int C, int cap, int *idx,
                        const ErrCtx &e, cudaStream_t stream) {
  switch (C) {
    case 1: return launch_c<1>(scores, ld, T, k, L, cap, idx, e, stream);
    case 2: return launch_c<2>(scores, ld, T, k, L, cap, idx, e, stream);
    case 4: return launch_c<4>(scores, ld, T, k, L, cap, idx, e, stream);
    case 8: return launch_c<8>(scores, ld, T, k, L, cap, idx, e, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dsa
