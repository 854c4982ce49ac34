// Fine-grained token selection from a filtered candidate list: the finishing
// half of an indexer -> top-k in which the indexer never writes its full score
// row (jdon.com "DeepSeek-V3.2-Exp", sparse-training and selection paragraphs:
// K = 2048 tokens kept per query).
//
// Input per query row: the histogram of the top 12 bits of the order key of
// every score s = 0..pos_t (complete), and a list of (score, position)
// candidates that holds at least every key whose bin is at or above the row's
// final threshold bin (the bin of the k-th best key). A producer gets this by
// appending each key whose bin is at or above any lower bound of that bin; a
// bound read from the histogram built so far is one, however stale.
//
// One CTA per row:
//   1. threshold bin B and the number of keys above it, from the histogram;
//   2. one pass over the candidates: keys above B go straight into a bitmap of
//      selected positions, keys in B into a tie list in shared memory;
//   3. the tie list is ranked exactly by (key descending, position ascending):
//      radix select on key bits 19..10 and 9..0, then on the position (18 bits)
//      among the keys equal to the threshold key (when bin B holds more keys
//      than shared memory stages, the passes read the candidate list instead);
//   4. the bitmap is emitted in ascending position order (a block scan of the
//      words' populations), then -1 padding.
// The result equals a full top-k over the row's scores: same order key (-0 and
// +0 equal, NaN lowest), same tie rule, same output order.
#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 4096;                   // top 12 bits of the order key
constexpr int kBinsPerThread = kBins / kThreads;
constexpr int kMaxPos = 262144;               // positions per row (bitmap bits)
constexpr int kWords = kMaxPos / 32;
constexpr int kTieCap = 12288;                // tie entries staged in shared memory
constexpr int kRadix = 1024;                  // bins of the later radix passes

// Same transform as the full top-k: larger float, larger key; -0 and +0 share a
// key; every NaN maps below -inf.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Shared {
  uint32_t bitmap[kWords];          // selected positions
  uint32_t tie_key[kTieCap];
  int tie_pos[kTieCap];
  unsigned cnt[4][kRadix];          // one histogram per radix pass (all cleared up front)
  unsigned warp_tot[kWarps];
  unsigned n_tie, n_above;
  int bin_b;                        // threshold bin
  unsigned above_b;                 // keys in bins above it (from the histogram)
  unsigned sel_digit, sel_rem, sel_cnt;  // result of a radix pass
  unsigned scan_total;              // block_exclusive's total
};

// Exclusive prefix of v over the block (thread order); *total gets the sum.
__device__ __forceinline__ unsigned block_exclusive(unsigned v, unsigned *total, Shared &sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm.warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const unsigned w = lane < kWarps ? sm.warp_tot[lane] : 0u;
    unsigned s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xFFFFFFFFu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kWarps) sm.warp_tot[lane] = s - w;  // exclusive over warps
    if (lane == 31) sm.scan_total = s;
  }
  __syncthreads();
  const unsigned ex = sm.warp_tot[warp] + x - v;
  *total = sm.scan_total;
  __syncthreads();                                // warp_tot and scan_total reusable
  return ex;
}

// One warp: among the counts c[0..kRadix), scanning from `from_top` ? the highest
// digit : the lowest, the digit d at which the running count reaches `need`. Writes
// d, the count strictly before d (in scan order) and c[d] to sm.sel_*.
__device__ __forceinline__ void find_digit_warp(const unsigned *c, unsigned need, bool from_top, Shared &sm) {
  const int lane = threadIdx.x & 31;
  constexpr int kPer = kRadix / 32;
  unsigned mine = 0;
#pragma unroll 8
  for (int j = 0; j < kPer; ++j) {  // lane l takes digits l*32 .. l*32+31 in scan order
    const int i = lane * kPer + j;
    mine += c[from_top ? kRadix - 1 - i : i];
  }
  unsigned incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  unsigned before = incl - mine;
  if (before < need && incl >= need) {  // the crossing lane walks its own digits again
    for (int j = 0; j < kPer; ++j) {
      const int i = lane * kPer + j;
      const int d = from_top ? kRadix - 1 - i : i;
      const unsigned v = c[d];
      if (before + v >= need) {
        sm.sel_digit = (unsigned)d;
        sm.sel_rem = before;
        sm.sel_cnt = v;
        break;
      }
      before += v;
    }
  }
}

struct CandParams {
  const float *score;     // [T][cap]
  const int *pos;         // [T][cap]
  const int *count;       // [T]
  long long cap;
  const unsigned *hist;   // [T][4096]
  int k;
  int *idx;               // [T][k]
  Layout L;
  ErrCtx e;
};

__global__ void __launch_bounds__(kThreads, 1) topk_candidates_kernel(const CandParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Shared &sm = *reinterpret_cast<Shared *>(smem_raw);
  pdl_prologue();
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int *out = p.idx + (long long)t * p.k;
  const RowPos rp = row_position(p.L, t);
  const long long n = (long long)rp.pos + 1;      // keys of the row
  if (rp.pos < 0 || n > kMaxPos || rp.len > cache_capacity(p.L)) {
    if (tid == 0) raise_error(p.e, DEV_BOUNDS, 0x900);
    for (int i = tid; i < p.k; i += kThreads) out[i] = -1;
    return;
  }
  const unsigned m = (unsigned)min((long long)p.k, n);
  const int nw = (int)((n + 31) >> 5);             // bitmap words in use
  // the row's histogram, this thread's 8 bins from the top down
  const unsigned *h = p.hist + (long long)t * kBins;
  const int b_hi = kBins - 1 - tid * kBinsPerThread;
  const uint4 ha = __ldg(reinterpret_cast<const uint4 *>(h + b_hi - 7));
  const uint4 hb = __ldg(reinterpret_cast<const uint4 *>(h + b_hi - 3));
  const unsigned hv[kBinsPerThread] = {hb.w, hb.z, hb.y, hb.x, ha.w, ha.z, ha.y, ha.x};
  for (int w = tid; w < nw; w += kThreads) sm.bitmap[w] = 0u;
  for (int i = tid; i < 4 * kRadix; i += kThreads) (&sm.cnt[0][0])[i] = 0u;
  if (tid == 0) {
    sm.n_tie = 0;
    sm.n_above = 0;
    sm.bin_b = -1;
  }

  // ---- 1. threshold bin: the highest b with at least m keys in bins >= b
  unsigned mine = 0;
#pragma unroll
  for (int j = 0; j < kBinsPerThread; ++j) mine += hv[j];
  unsigned total;
  unsigned above = block_exclusive(mine, &total, sm);  // keys in bins above this thread's
  if (total < m) {  // the histogram does not count the row's keys
    if (tid == 0) raise_error(p.e, DEV_BOUNDS, 0x901);
    for (int i = tid; i < p.k; i += kThreads) out[i] = -1;
    return;
  }
#pragma unroll
  for (int j = 0; j < kBinsPerThread; ++j) {
    if (above < m && above + hv[j] >= m) {
      sm.bin_b = b_hi - j;
      sm.above_b = above;
    }
    above += hv[j];
  }
  __syncthreads();
  const int B = sm.bin_b;
  const unsigned need_ties = m - sm.above_b;  // entries to take from bin B (>= 1)

  // ---- 2. sort the candidates into "above B" (selected) and "in B" (ties)
  long long cnt = p.count[t];
  if (cnt > p.cap) {
    if (tid == 0) raise_error(p.e, DEV_BOUNDS, 0x902);
    cnt = p.cap;
  }
  const float *cs = p.score + (long long)t * p.cap;
  const int *cp = p.pos + (long long)t * p.cap;
  const unsigned lt = (1u << lane) - 1u;
  // Every lane of a warp runs the same iterations. Each lane loads kU candidates
  // before it looks at any, so that the loads' latencies overlap; a warp reserves
  // its ties' slots with one shared-memory atomic per kU x 32 candidates, and the
  // keys above B are counted per thread and summed once at the end.
  constexpr int kU = 8;
  unsigned my_above = 0;
  for (long long i0 = (long long)(tid - lane) * kU; i0 < cnt; i0 += (long long)kThreads * kU) {
    float sc[kU];
    int ps[kU];
#pragma unroll
    for (int j = 0; j < kU; ++j) {
      const long long i = i0 + j * 32 + lane;
      sc[j] = i < cnt ? __ldg(cs + i) : 0.f;
      ps[j] = i < cnt ? __ldg(cp + i) : 0;
    }
    unsigned tie_bits = 0, tmask[kU], n_tie_w = 0;
#pragma unroll
    for (int j = 0; j < kU; ++j) {
      const long long i = i0 + j * 32 + lane;
      const uint32_t key = order_key(sc[j]);
      const int s = ps[j];
      bool is_above = false, is_tie = false;
      if (i < cnt) {
        const int bin = (int)(key >> 20);
        if (bin >= B) {
          if (s < 0 || (long long)s >= n) {
            raise_error(p.e, DEV_BOUNDS, 0x903);
          } else {
            is_above = bin > B;
            is_tie = bin == B;
          }
        }
      }
      if (is_above) atomicOr(&sm.bitmap[s >> 5], 1u << (s & 31));
      my_above += is_above;
      tmask[j] = __ballot_sync(0xFFFFFFFFu, is_tie);
      tie_bits |= (unsigned)is_tie << j;
      n_tie_w += __popc(tmask[j]);
    }
    if (n_tie_w) {
      unsigned tb = 0;
      if (lane == 0) tb = atomicAdd(&sm.n_tie, n_tie_w);
      tb = __shfl_sync(0xFFFFFFFFu, tb, 0);
#pragma unroll
      for (int j = 0; j < kU; ++j) {
        if ((tie_bits >> j) & 1u) {
          const unsigned slot = tb + __popc(tmask[j] & lt);
          if (slot < kTieCap) {
            sm.tie_key[slot] = order_key(sc[j]);
            sm.tie_pos[slot] = ps[j];
          }
        }
        tb += __popc(tmask[j]);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) my_above += __shfl_xor_sync(0xFFFFFFFFu, my_above, o);
  if (lane == 0 && my_above) atomicAdd(&sm.n_above, my_above);
  __syncthreads();
  const unsigned n_tie = sm.n_tie;
  // every key in bins >= B must have been a candidate: the counts must agree
  if (sm.n_above != sm.above_b || n_tie != h[B]) {
    if (tid == 0) raise_error(p.e, DEV_BOUNDS, 0x904);
    for (int i = tid; i < p.k; i += kThreads) out[i] = -1;
    return;
  }

  // ---- 3. exact ranking inside bin B: key bits 19..10, 9..0, then (only when
  // more keys equal the threshold key than are taken) the position, lowest first
  const bool staged = n_tie <= kTieCap;
  auto for_ties = [&](auto f) {  // every (key, position) of bin B, this thread's share
    if (staged) {
      for (unsigned i = tid; i < n_tie; i += kThreads) f(sm.tie_key[i], sm.tie_pos[i]);
    } else {
      for (long long i = tid; i < cnt; i += kThreads) {
        const uint32_t key = order_key(__ldg(cs + i));
        if ((int)(key >> 20) == B) f(key, __ldg(cp + i));
      }
    }
  };
  uint32_t kstar = 0;       // threshold key
  int pstar = kMaxPos - 1;  // largest selected position among keys equal to kstar
  if (need_ties < n_tie) {
    uint32_t prefix = (uint32_t)B << 20;
    unsigned need = need_ties, at_kstar = 0;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 10 : 0;
      const uint32_t pmask = pass == 0 ? 0xFFF00000u : 0xFFFFFC00u;
      unsigned *c = sm.cnt[pass];
      for_ties([&](uint32_t key, int) {
        if ((key & pmask) == prefix) atomicAdd(&c[(key >> shift) & (kRadix - 1)], 1u);
      });
      __syncthreads();
      if (warp == 0) find_digit_warp(c, need, true, sm);
      __syncthreads();
      prefix |= sm.sel_digit << shift;
      need -= sm.sel_rem;
      at_kstar = sm.sel_cnt;
    }
    kstar = prefix;  // need = how many keys equal to kstar are taken (lowest positions first)
    if (need < at_kstar) {
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {  // positions < 2^18 in two 9-bit digits
        const int shift = pass == 0 ? 9 : 0;
        unsigned *c = sm.cnt[2 + pass];
        const int phi = pstar >> 9;
        for_ties([&](uint32_t key, int s) {
          const bool in = key == kstar && (pass == 0 || (s >> 9) == phi);
          if (in) atomicAdd(&c[(s >> shift) & 511], 1u);
        });
        __syncthreads();
        if (warp == 0) find_digit_warp(c, need, false, sm);
        __syncthreads();
        if (pass == 0) {
          pstar = (int)(sm.sel_digit << 9) | 511;
        } else {
          pstar = (pstar & ~511) | (int)sm.sel_digit;
        }
        need -= sm.sel_rem;
      }
    }
  } else {
    kstar = 0;  // every tie is taken
  }
  for_ties([&](uint32_t key, int s) {
    if (need_ties >= n_tie || key > kstar || (key == kstar && s <= pstar))
      atomicOr(&sm.bitmap[s >> 5], 1u << (s & 31));
  });
  __syncthreads();

  // ---- 4. ascending emission, then padding. Warp w takes a contiguous block of
  // bitmap words, 32 at a time (one per lane): its total first, then, after a scan
  // of the warps' totals, each lane writes its word's positions at its prefix.
  const int per_w = (nw + kWarps - 1) / kWarps;
  const int wb0 = min(nw, warp * per_w), wb1 = min(nw, wb0 + per_w);
  unsigned wt = 0;
  for (int w = wb0 + lane; w < wb1; w += 32) wt += __popc(sm.bitmap[w]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wt += __shfl_xor_sync(0xFFFFFFFFu, wt, o);
  if (lane == 0) sm.warp_tot[warp] = wt;
  __syncthreads();
  if (warp == 0) {
    const unsigned v = lane < kWarps ? sm.warp_tot[lane] : 0u;
    unsigned incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane < kWarps) sm.warp_tot[lane] = incl - v;
    if (lane == 31) sm.scan_total = incl;
  }
  __syncthreads();
  const unsigned emitted = sm.scan_total;
  if (emitted != m && tid == 0) raise_error(p.e, DEV_BOUNDS, 0x905);
  unsigned base = sm.warp_tot[warp];
  for (int w0 = wb0; w0 < wb1; w0 += 32) {
    const int w = w0 + lane;
    uint32_t bits = w < wb1 ? sm.bitmap[w] : 0u;
    const unsigned c = __popc(bits);
    unsigned incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    unsigned off = base + incl - c;
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      if (off < (unsigned)p.k) out[off] = w * 32 + bit;
      ++off;
    }
    base += __shfl_sync(0xFFFFFFFFu, incl, 31);
  }
  for (int i = (int)emitted + tid; i < p.k; i += kThreads) out[i] = -1;
}

}  // namespace

size_t topk_candidates_smem() { return sizeof(Shared); }

cudaError_t launch_topk_candidates(const float *score, const int *pos, const int *count, long long cap,
                                   const unsigned *hist, int T, int k, const Layout &L, int *idx, const ErrCtx &e,
                                   cudaStream_t stream) {
  const size_t smem = sizeof(Shared);
  cudaError_t err = cudaFuncSetAttribute(topk_candidates_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  CandParams p;
  p.score = score;
  p.pos = pos;
  p.count = count;
  p.cap = cap;
  p.hist = hist;
  p.k = k;
  p.idx = idx;
  p.L = L;
  p.e = e;
  return launch_kernel(topk_candidates_kernel, dim3(T), dim3(kThreads), smem, stream, 0, p);
}

}  // namespace dsa
