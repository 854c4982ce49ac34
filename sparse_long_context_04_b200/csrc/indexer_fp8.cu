// Lightning indexer on the 5th-generation tensor cores (FP8 e4m3, tcgen05).
//
//   I[t,s] = s_q[t] * s_k[s] * sum_j w[t,j] * max(0, dec(q8[t,j,:]) . dec(k8[s,:]))
//
// jdon.com "DeepSeek-V3.2-Exp": the indexer is light enough to run in FP8 with
// very few heads and scores each query token against each earlier token with a
// weighted sum of ReLU-activated dot products (w_I the weight). The per-token
// scales are positive, so ReLU(s_q s_k x) = s_q s_k ReLU(x) and they are applied
// once per output.
//
// One MMA tile: D[128 keys, 64*G] = K8[128 keys, 128] . Q8[G tokens x 64 heads, 128]^T
// (kind::f8f6f4, M = 128, N = 64G, K = 128 as four K = 32 steps), accumulated in
// TMEM. The epilogue reads each key's row of D, applies ReLU, weights by w[t,:]
// and sums the 64 heads of each token in registers, so the [t, j, s] tensor never
// leaves the SM. G = 1 serves decode (one query per sequence); G = 4 serves
// prefill (four consecutive query tokens of a sequence share each key tile).
//
// Work: the flat list of (query group, key tile) items of every sequence, key
// tiles 0 .. floor(last position / 128) per group (causal), is split into one
// contiguous range per persistent CTA. Item counts have a closed form, so each
// CTA finds its range without a pre-pass.
//
// Roles: four producer warps take every fourth tile and issue its TMA loads (keys
// as two 64-row boxes, one per page in a paged cache, plus the keys' fp32 scales
// by bulk copy; for a new query group also the group's query box and weights),
// so several tiles are always being requested; two MMA warps take alternate tiles
// and issue their MMAs into separate TMEM accumulators (one issuing thread cannot
// keep up with HBM: each tile needs waits, four MMAs and two commits); eight warps
// run the epilogue (decode: two groups of four take alternate tiles; prefill: all
// eight, two query tokens each).
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int kHI = 64;      // indexer heads
constexpr int kDI = 128;     // indexer dim (bytes per e4m3 row)
constexpr int kTileKeys = 128;

template <int G>
struct Cfg {
  static constexpr int N = kHI * G;
  static constexpr int kStages = G == 1 ? 8 : 4;
  static constexpr int kProdWarps = 4;                  // tile n is issued by producer warp n % 4
  static constexpr int kMmaWarps = 2;                   // tile n's MMAs are issued by MMA warp n % 2
  static constexpr int kMmaWarp0 = kProdWarps;
  static constexpr int kEpiWarp0 = kProdWarps + kMmaWarps;
  static constexpr int kEpiWarps = 8;
  static constexpr int kWarpsPerItem = G == 1 ? 4 : 8;  // decode: two groups of four warps alternate tiles
  static constexpr int kAccBufs = G == 1 ? 8 : 2;       // TMEM accumulators (N columns each)
  static constexpr int kBoundWarp = kProdWarps + kMmaWarps + kEpiWarps;  // decode: the fused top-k's bound
  static constexpr int kThreads = 32 * (kProdWarps + kMmaWarps + kEpiWarps + (G == 1 ? 1 : 0));
  static constexpr int kATile = kTileKeys * kDI;  // 16 KiB
  static constexpr int kBTile = N * kDI;          // 8 or 32 KiB
  static constexpr int kWBytes = G * kHI * 4;     // head weights of a query group
  static constexpr int kTmemCols = kAccBufs * N;  // 512
  static constexpr int kData = kStages * kATile + 2 * kBTile + kStages * kTileKeys * 4 + 2 * kWBytes;
  static constexpr int kSmem = 1024 + kData + 1024;  // alignment slack + barriers
  static constexpr uint32_t kIdesc = instr_desc(0, 0, 0, 0, 128, N);
  static_assert(kStages % kProdWarps == 0, "each producer warp owns whole stages");
};

struct Params {
  const float *q_scale;   // [T]
  const float *k_scale;   // contiguous [B][n_max]; nullptr when paged
  const uint8_t *k_pool;  // paged pool base (scales live in the pages)
  const float *w;         // [T][64]
  int scales_bulk;        // key scales reach shared memory by bulk copy (else read per thread)
  float *scores;          // [T][ld] (unless fuse)
  // fused top-k (decode): instead of the scores, per row the candidates (keys at
  // or above a lower bound of the row's threshold bin) and their histogram by the
  // top 12 bits of the order key
  int fuse;
  int k;
  unsigned *hist;         // [T][4096], zero at launch, 16-byte aligned
  int *cand_count;        // [T], zero at launch
  float *cand_score;      // [T][cand_cap]
  int *cand_pos;          // [T][cand_cap]
  long long cand_cap;
  long long ld;
  int T;
  Layout L;
  ErrCtx e;
};

// ------------------------------------------------------------------ work walk
// Rows of sequence b inside this launch, grouped G at a time from the first.
struct SeqRows {
  int Qc;              // query rows of the sequence in this launch (0 = none)
  int r_lo;            // first local row
  long long p_first;   // position of that row
  int len;             // keys of the sequence
};

__device__ __forceinline__ SeqRows seq_rows(const Params &p, int b) {
  SeqRows s;
  const Layout &L = p.L;
  s.len = __ldg(L.seq_lens + b);
  s.Qc = 0;
  s.r_lo = 0;
  s.p_first = 0;
  long long g_lo, g_hi, q0, Q;
  if (L.cu_q == nullptr) {
    q0 = b;
    Q = 1;
  } else {
    q0 = __ldg(L.cu_q + b);
    Q = __ldg(L.cu_q + b + 1) - q0;
  }
  g_lo = max(q0, (long long)L.row0);
  g_hi = min(q0 + Q, (long long)L.row0 + p.T);
  if (g_hi <= g_lo) return s;
  if (s.len < 1 || s.len > cache_capacity(L) || Q > s.len) {
    raise_error(p.e, DEV_BOUNDS, 0x400);
    return s;
  }
  s.Qc = (int)(g_hi - g_lo);
  s.r_lo = (int)(g_lo - L.row0);
  s.p_first = s.len - Q + (g_lo - q0);
  return s;
}

// F(n) = sum_{v=0}^{n-1} floor(v / P)
__device__ __forceinline__ long long floor_prefix(long long n, long long P) {
  const long long q = n / P, r = n % P;
  return P * q * (q - 1) / 2 + q * r;
}

template <int G>
struct GroupMath {
  // key tiles of the first i groups of a sequence (all of them full groups)
  __device__ static long long tiles_before(const SeqRows &s, long long i) {
    const long long P = kTileKeys / G;
    const long long u0 = (s.p_first + G - 1) / G;
    return i + floor_prefix(u0 + i, P) - floor_prefix(u0, P);
  }
  __device__ static int groups(const SeqRows &s) { return (s.Qc + G - 1) / G; }
  __device__ static long long last_pos(const SeqRows &s, int i) {
    return min(s.p_first + (long long)(i + 1) * G - 1, s.p_first + s.Qc - 1);
  }
  __device__ static int tiles_of(const SeqRows &s, int i) { return (int)(last_pos(s, i) / kTileKeys) + 1; }
  __device__ static long long tiles_total(const SeqRows &s) {
    if (s.Qc == 0) return 0;
    const int ng = groups(s);
    return tiles_before(s, ng - 1) + tiles_of(s, ng - 1);
  }
};

// A cursor over this CTA's items (in order). Every role steps its own copy.
template <int G>
struct Cursor {
  int b, i, kt, ntiles, ng;
  int gcount;      // query groups started so far in this CTA's range, the current one included
  SeqRows s;
  long long left;  // items from the current one to the end of the range, the current one included

  __device__ void enter_seq(const Params &p, int nb) {
    b = nb;
    s = seq_rows(p, b);
    ng = GroupMath<G>::groups(s);
  }
  // position at flat item f of sequence b (0 <= f < tiles_total)
  __device__ void seek(const Params &p, int nb, long long f, long long count) {
    enter_seq(p, nb);
    int lo = 0, hi = ng - 1;  // largest i with tiles_before(i) <= f
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (GroupMath<G>::tiles_before(s, mid) <= f) lo = mid; else hi = mid - 1;
    }
    i = lo;
    kt = (int)(f - GroupMath<G>::tiles_before(s, i));
    ntiles = GroupMath<G>::tiles_of(s, i);
    left = count;
    gcount = 1;
  }
  // step one item; true when the new item starts a query group
  __device__ bool next(const Params &p) {
    --left;
    if (left <= 0) return false;
    if (++kt < ntiles) return false;
    kt = 0;
    ++gcount;
    if (++i >= ng) {
      i = 0;
      do {
        enter_seq(p, b + 1);
      } while (ng == 0 && b + 1 < p.L.batch);
    }
    ntiles = GroupMath<G>::tiles_of(s, i);
    return true;
  }
  // step k >= 1 items
  __device__ void advance(const Params &p, int k) {
    if (kt + k < ntiles && left > k) {
      kt += k;
      left -= k;
      return;
    }
    for (int j = 0; j < k; ++j) next(p);
  }
  __device__ int row0() const { return s.r_lo + i * G; }
  __device__ int rows() const { return min(G, s.Qc - i * G); }
};

// One tile of a producer warp's 32-tile batch, held by the lane of the same index.
struct Item {
  int b, kt, row0;
  int gslot;          // query group's B slot (0/1) | 2 if the tile starts the group | use count << 2
  int pg0, pg1, has1;  // paged: physical pages of the tile's two 64-key halves
};

// Producer warp: walks the next (up to) 32 of its tiles — this warp's tiles are
// every kProdWarps-th item — and has lane j keep tile j; for a paged cache each
// lane starts loading its page ids. `n` is the item index of the cursor.
template <int G>
__device__ __forceinline__ int collect_batch(const Params &p, Cursor<G> &cur, long long &n, long long n_items,
                                             int lane, Item &it) {
  using C = Cfg<G>;
  it.b = 0;
  it.kt = 0;
  it.row0 = 0;
  it.gslot = 0;
  it.pg0 = -1;
  it.pg1 = -1;
  it.has1 = 0;
  int cnt = 0, len = 0;
  for (int j = 0; j < 32 && n < n_items; ++j) {
    if (lane == j) {
      it.b = cur.b;
      it.kt = cur.kt;
      it.row0 = cur.row0();
      const int g = cur.gcount - 1;
      it.gslot = (g & 1) | ((cur.kt == 0 || n == 0) ? 2 : 0) | ((g >> 1) << 2);
      len = cur.s.len;
    }
    ++cnt;
    n += C::kProdWarps;
    if (n < n_items) cur.advance(p, C::kProdWarps);
  }
  if (p.L.page_size && lane < cnt) {
    const int *pt = p.L.page_table + (long long)it.b * p.L.max_pages + it.kt * 2;
    it.pg0 = __ldg(pt);
    it.has1 = it.kt * kTileKeys + 64 < len;
    if (it.has1) it.pg1 = __ldg(pt + 1);
  }
  return cnt;
}

// ------------------------------------------------------------------ fused top-k helpers
// Order key of a score (the selection's rule): larger float, larger key; -0 and
// +0 share a key; every NaN maps below -inf. Its top 12 bits are the row
// histogram's bin, its top 6 bits the coarse bin.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// A lower bound on row t's final threshold bin (the bin of its k-th best key),
// not below `cur` (the previous one): the highest bin with at least k candidates
// at or above it in the candidates' histogram as it stands. Only bins at or above
// the current bound are counted (keys below it are not candidates), and a later
// bound can only be higher, so the bins below it never matter again. Each count
// read is at most its final value and at most the row's number of scores in that
// bin, so the bin found has at least k of the row's keys at or above it in the
// end. Bins above `top` (the highest candidate bin this CTA has seen in the row)
// are not read: leaving counts out only lowers the bound. One warp: a pass over
// bins [cur rounded down to 128, top rounded up), then the bins of the lane where
// the count crosses k.
__device__ int row_bound(const Params &p, int t, int cur, int top) {
  const int lane = threadIdx.x & 31;
  const unsigned k = (unsigned)p.k;
  const unsigned *hf = p.hist + (long long)t * 4096;
  const int lo = cur & ~127;
  const int nb = min(4096 - lo, (max(top + 1 - lo, 1) + 127) & ~127);  // a multiple of 128
  const int per = nb >> 5;  // bins per lane: a multiple of 4, 4..128
  const int b0 = lo + lane * per;    // this lane's bins [b0, b0 + per)
  unsigned mine = 0;
  for (int j = 0; j < per; j += 4) {
    const uint4 v = __ldcg(reinterpret_cast<const uint4 *>(hf + b0 + j));
    mine += v.x + v.y + v.z + v.w;
  }
  unsigned suf = mine;  // candidates in this lane's bins and those of the lanes above
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_down_sync(0xFFFFFFFFu, suf, o);
    if (lane + o < 32) suf += y;
  }
  const unsigned hit = __ballot_sync(0xFFFFFFFFu, suf - mine < k && suf >= k);
  if (!hit) return cur;  // fewer than k counted in the window so far
  const int src = __ffs(hit) - 1;
  const int hi = __shfl_sync(0xFFFFFFFFu, b0, src) + per - 1;  // highest bin of the crossing lane
  unsigned run = __shfl_sync(0xFFFFFFFFu, suf - mine, src);     // candidates above `hi`
  for (int c0 = 0; c0 < per; c0 += 32) {
    const int bin = hi - c0 - lane;
    const unsigned cnt = c0 + lane < per ? __ldcg(hf + bin) : 0u;
    unsigned incl = cnt;  // this bin and the higher ones of this chunk
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    const unsigned f = __ballot_sync(0xFFFFFFFFu, run + incl - cnt < k && run + incl >= k);
    if (f) return max(cur, __shfl_sync(0xFFFFFFFFu, bin, __ffs(f) - 1));
    run += __shfl_sync(0xFFFFFFFFu, incl, 31);
  }
  return cur;  // the lane's bins grew after the first pass; keep the bound
}

// ------------------------------------------------------------------ kernel
// F: the fused top-k's producer (decode only) instead of score rows; PG: the key
// cache is paged (its scales always come by bulk copy). Template arguments so that
// each kernel carries only its own branches and state.
template <int G, bool F, bool PG>
__global__ void __launch_bounds__(Cfg<G>::kThreads, 1)
    indexer_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const Params p) {
  using C = Cfg<G>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char *base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  unsigned char *sA = base;
  unsigned char *sB = base + C::kStages * C::kATile;
  float *sScale = reinterpret_cast<float *>(sB + 2 * C::kBTile);       // [stage][128] key scales
  float *sW = sScale + C::kStages * kTileKeys;                         // [slot][G][64] head weights
  uint64_t *bars = reinterpret_cast<uint64_t *>(base + C::kData);
  uint64_t *a_full = bars, *a_empty = bars + C::kStages;
  uint64_t *b_full = bars + 2 * C::kStages, *b_empty = b_full + 2;
  uint64_t *acc_full = b_empty + 2, *acc_empty = acc_full + C::kAccBufs;
  uint64_t *done_bar = acc_empty + C::kAccBufs;  // one per MMA warp
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done_bar + C::kMmaWarps);
  __shared__ long long s_range[2];  // first flat item of this CTA, number of items
  __shared__ int s_seq;             // sequence holding the first item
  __shared__ long long s_fseq;      // flat index of the first item within that sequence
  __shared__ int s_b_turn;          // query-group loads issued so far (they are issued in group order)
  __shared__ unsigned long long s_bound;  // fused top-k: (row << 32) | lower bound of that row's threshold bin
  __shared__ unsigned long long s_top;    // fused top-k: (row << 32) | highest candidate bin seen in that row
  __shared__ int s_cur_row;               // fused top-k: the row the epilogue is scoring (-1: none yet)
  __shared__ int s_tiles;                 // fused top-k: tiles the epilogue has finished
  __shared__ int s_epi_done;              // fused top-k: epilogue warps that have finished

  pdl_prologue();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = p.L.batch;

  // ---- barriers and TMEM (independent of the work range, so set up while its loads run)
  if (threadIdx.x == 0) {
    for (int st = 0; st < C::kStages; ++st) {
      mbar_init(a_full + st, 1);
      mbar_init(a_empty + st, 1 + C::kWarpsPerItem);  // the MMA commit and the tile's epilogue warps
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(b_full + j, 1);
      mbar_init(b_empty + j, C::kMmaWarps + C::kEpiWarps);  // every MMA and epilogue warp
    }
    for (int j = 0; j < C::kAccBufs; ++j) {
      mbar_init(acc_full + j, 1);
      mbar_init(acc_empty + j, C::kWarpsPerItem);
    }
    for (int j = 0; j < C::kMmaWarps; ++j) mbar_init(done_bar + j, 1);
    s_b_turn = 0;
    s_bound = 0ull;
    s_top = 0ull;
    s_cur_row = -1;
    s_tiles = 0;
    s_epi_done = 0;
    fence_mbar_init();
  }
  if (warp == C::kMmaWarp0) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  // ---- work range: per-sequence item counts (closed form), block prefix sum
  {
    long long *pre = reinterpret_cast<long long *>(sA);  // aliases stage memory before any load
    __shared__ long long part[32];
    const int per = (B + blockDim.x - 1) / blockDim.x;
    const int b0 = threadIdx.x * per, b1 = min(B, b0 + per);
    long long acc = 0;
    for (int b = b0; b < b1; ++b) {
      const SeqRows sr = seq_rows(p, b);
      const long long n = GroupMath<G>::tiles_total(sr);
      pre[b] = n;
      acc += n;
    }
    long long incl = acc;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) part[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int nw = blockDim.x >> 5;
      long long v = lane < nw ? part[lane] : 0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const long long o = __shfl_up_sync(0xFFFFFFFFu, v, off);
        if (lane >= off) v += o;
      }
      if (lane < nw) part[lane] = v;  // inclusive per-warp totals
    }
    __syncthreads();
    long long run = (warp ? part[warp - 1] : 0) + incl - acc;
    for (int b = b0; b < b1; ++b) {
      const long long n = pre[b];
      pre[b] = run;
      run += n;
    }
    const long long W = part[(blockDim.x >> 5) - 1];
    __syncthreads();
    if (threadIdx.x == 0) {
      const long long f0 = W * blockIdx.x / gridDim.x;
      const long long f1 = W * (blockIdx.x + 1) / gridDim.x;
      int lo = 0, hi = B - 1;  // last sequence with pre[b] <= f0
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= f0) lo = mid; else hi = mid - 1;
      }
      s_seq = lo;
      s_fseq = f0 - pre[lo];
      s_range[0] = f0;
      s_range[1] = f1 - f0;
      if (G == 1 && p.L.page_size && p.L.cu_q == nullptr) {
        // decode: this CTA's items are key tiles s_fseq.. of sequence lo, two page ids each;
        // start the page-table reads now so that they overlap the set-up below
        const int *row = p.L.page_table + (long long)lo * p.L.max_pages;
        const long long e0 = 2 * s_fseq;
        const long long e1 = min((long long)p.L.max_pages, e0 + 2 * (f1 - f0));
        for (long long e = e0 & ~31ll; e < e1 && e < e0 + 256; e += 32) prefetch_l2(row + e);
      }
    }
    __syncthreads();
  }
  const long long n_items = s_range[1];
  tc_fence_after();  // the work range's block barriers also ordered the TMEM allocation
  const uint32_t tmem = *tmem_slot;

  if (n_items > 0) {
    if (warp < C::kProdWarps) {
      // ================= producer warps: tiles n with n % kProdWarps == warp
      if (warp < n_items) {
        if (lane == 0) {
          tma_prefetch_desc(&tm_q);
          tma_prefetch_desc(&tm_k);
        }
        Cursor<G> cur;
        cur.seek(p, s_seq, s_fseq, n_items);
        if (warp > 0) cur.advance(p, warp);
        long long n_walk = warp;         // item the cursor is at
        long long n_issue = warp;        // next item to issue
        bool ok = true;
        Item nxt;
        int ncnt = collect_batch<G>(p, cur, n_walk, n_items, lane, nxt);
        while (ncnt > 0 && ok) {
          const Item it = nxt;
          const int cnt = ncnt;
          ncnt = n_walk < n_items ? collect_batch<G>(p, cur, n_walk, n_items, lane, nxt) : 0;
          for (int j = 0; j < cnt; ++j, n_issue += C::kProdWarps) {
            const int b = __shfl_sync(0xFFFFFFFFu, it.b, j);
            const int kt = __shfl_sync(0xFFFFFFFFu, it.kt, j);
            const int row0 = __shfl_sync(0xFFFFFFFFu, it.row0, j);
            const int gs = __shfl_sync(0xFFFFFFFFu, it.gslot, j);
            const int pg0 = __shfl_sync(0xFFFFFFFFu, it.pg0, j);
            const int pg1 = __shfl_sync(0xFFFFFFFFu, it.pg1, j);
            const int has1 = __shfl_sync(0xFFFFFFFFu, it.has1, j);
            if (lane == 0) {
              if (gs & 2) {  // first tile of a query group: its queries and weights
                const int slot = gs & 1, use = gs >> 2;
                // groups are loaded in order (one producer warp after another), so that
                // each parity wait on a slot follows the wait for that slot's previous use
                ok = wait_turn(&s_b_turn, use * 2 + slot, p.e, 0x415);
                if (ok) ok = mbar_wait(b_empty + slot, (use & 1) ^ 1, p.e, 0x410);
                if (ok) {
                  const int nrow = min(G, p.T - row0);
                  mbar_expect_tx(b_full + slot, C::kBTile + nrow * kHI * 4);
                  tma_load_2d(sB + slot * C::kBTile, &tm_q, b_full + slot, 0, row0 * kHI);
                  bulk_load(sW + slot * G * kHI, p.w + (long long)row0 * kHI, nrow * kHI * 4, b_full + slot);
                  __threadfence_block();
                  *reinterpret_cast<volatile int *>(&s_b_turn) = use * 2 + slot + 1;
                }
              }
              const int st = (int)(n_issue % C::kStages);
              const uint32_t use = (uint32_t)(n_issue / C::kStages);
              if (ok) ok = mbar_wait(a_empty + st, (use & 1) ^ 1, p.e, 0x411);
              if (ok) {
                const int s0 = kt * kTileKeys;
                unsigned char *dst = sA + st * C::kATile;
                float *sdst = sScale + st * kTileKeys;
                int y0 = -1, y1 = -1;
                const unsigned char *sc0 = nullptr, *sc1 = nullptr;
                uint32_t sb0 = 0, sb1 = 0;
                if (!PG) {
                  y0 = (int)((long long)b * p.L.n_max + s0);
                  y1 = y0 + 64;
                  if (p.scales_bulk) {
                    sc0 = reinterpret_cast<const unsigned char *>(p.k_scale + (long long)b * p.L.n_max + s0);
                    sb0 = (uint32_t)min(kTileKeys, p.L.n_max - s0) * 4u;
                  }
                } else {
                  const bool ok0 = (unsigned)pg0 < (unsigned)p.L.num_pages;
                  const bool ok1 = has1 && (unsigned)pg1 < (unsigned)p.L.num_pages;
                  if (!ok0 || (has1 && !ok1)) raise_error(p.e, DEV_BOUNDS, 0x412);
                  if (ok0) {
                    y0 = pg0 * 66;
                    sc0 = p.k_pool + (long long)pg0 * 8448 + 8192;
                    sb0 = 256;
                  }
                  if (ok1) {
                    y1 = pg1 * 66;
                    sc1 = p.k_pool + (long long)pg1 * 8448 + 8192;
                    sb1 = 256;
                  }
                }
                mbar_expect_tx(a_full + st, (y0 >= 0 ? 8192u : 0u) + (y1 >= 0 ? 8192u : 0u) + sb0 + sb1);
                if (y0 >= 0) tma_load_2d(dst, &tm_k, a_full + st, 0, y0);
                if (y1 >= 0) tma_load_2d(dst + 8192, &tm_k, a_full + st, 0, y1);
                if (sb0) bulk_load(sdst, sc0, sb0, a_full + st);
                if (sb1) bulk_load(sdst + 64, sc1, sb1, a_full + st);
              }
            }
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
            if (!ok) break;
          }
        }
        if (lane == 0) {
          // no copy may still be landing in shared memory at exit: wait for the last
          // tile this warp issued into each of its own stages (query slots: MMA warp)
          const long long issued_end = n_issue;  // one past this warp's last issued item (stride kProdWarps)
          for (int k = 1; k <= C::kStages / C::kProdWarps; ++k) {
            const long long n_last = issued_end - (long long)k * C::kProdWarps;
            if (n_last >= warp) mbar_wait(a_full + n_last % C::kStages, (uint32_t)(n_last / C::kStages) & 1, p.e, 0x413);
          }
        }
      }
      __syncwarp();
    } else if (warp < C::kEpiWarp0) {
      // ================= MMA warps (one lane each): tiles n with n % kMmaWarps == mw
      const int mw = warp - C::kMmaWarp0;
      if (lane == 0) {
        Cursor<G> cur;
        cur.seek(p, s_seq, s_fseq, n_items);
        int g_seen = 0;  // query groups whose slot this warp has waited for
        bool ok = true;
        // descriptors built once: a stage, query slot or K step moves only the start
        // address field (16-byte units; shared addresses stay below 2^18, so adding
        // an offset never carries out of the field)
        const uint64_t a_desc0 = smem_desc(smem_u32(sA), 16, 1024, SW_128B);
        const uint64_t b_desc0 = smem_desc(smem_u32(sB), 16, 1024, SW_128B);
        for (long long n = 0; n < n_items && ok; ++n) {
          const int g = cur.gcount - 1;
          const int slot = g & 1;
          if ((int)(n % C::kMmaWarps) == mw) {
            if (g_seen <= g) {
              ok = mbar_wait(b_full + slot, (uint32_t)(g >> 1) & 1, p.e, 0x420);
              if (!ok) break;
              g_seen = g + 1;
            }
            const int st = (int)(n % C::kStages);
            const uint32_t use = (uint32_t)(n / C::kStages);
            const int ab = (int)(n % C::kAccBufs);
            ok = mbar_wait(a_full + st, use & 1, p.e, 0x421);
            if (!ok) break;
            ok = mbar_wait(acc_empty + ab, ((uint32_t)(n / C::kAccBufs) & 1) ^ 1, p.e, 0x422);
            if (!ok) break;
            tc_fence_after();
            const uint32_t d = tmem + (uint32_t)(ab * C::N);
            const uint64_t ad = a_desc0 + (uint64_t)((st * C::kATile) >> 4);
            const uint64_t bd = b_desc0 + (uint64_t)((slot * C::kBTile) >> 4);
#pragma unroll
            for (int ks = 0; ks < kDI / 32; ++ks) umma_f8(d, ad + 2 * ks, bd + 2 * ks, C::kIdesc, ks > 0);
            umma_commit(a_empty + st);
            umma_commit(acc_full + ab);
          }
          // leaving group g: this warp's MMAs on the group's query slot are issued
          if (cur.next(p) || n + 1 == n_items) umma_commit(b_empty + slot);
        }
        umma_commit(done_bar + mw);
        mbar_wait(done_bar + mw, 0, p.e, 0x423);
        if (mw == 0) {
          // the query loads of the last two groups are the latest phases of the two slots
          const int g_last = cur.gcount - 1;
          for (int g = max(0, g_last - 1); g <= g_last; ++g)
            mbar_wait(b_full + (g & 1), (uint32_t)(g >> 1) & 1, p.e, 0x424);
        }
      }
      __syncwarp();
    } else if (G == 1 && warp == C::kBoundWarp) {
      // ================= bound warp (fused top-k): about once a microsecond, a fresh
      // lower bound of the current row's threshold bin from the global histograms
      if (F) {
        const unsigned long long t0 = globaltimer();
        int seen = -1;  // tiles finished at the last refresh: refresh only after new ones
        while (*reinterpret_cast<volatile int *>(&s_epi_done) < C::kEpiWarps) {
          const int row = *reinterpret_cast<volatile int *>(&s_cur_row);
          const int tiles = *reinterpret_cast<volatile int *>(&s_tiles);
          if (row >= 0 && tiles != seen) {
            seen = tiles;
            const unsigned long long old = *reinterpret_cast<volatile unsigned long long *>(&s_bound);
            const unsigned long long tp = *reinterpret_cast<volatile unsigned long long *>(&s_top);
            const int bnd = row_bound(p, row, (int)(old >> 32) == row ? (int)(unsigned)old : 0,
                                      (int)(tp >> 32) == row ? (int)(unsigned)tp : 4095);
            if (lane == 0)
              *reinterpret_cast<volatile unsigned long long *>(&s_bound) =
                  ((unsigned long long)(unsigned)row << 32) | (unsigned)bnd;
          }
          __syncwarp();
          __nanosleep(1000);
          if (error_raised(p.e)) break;
          if (globaltimer() - t0 > p.e.limit) {  // the epilogue never finished: give up
            if (lane == 0) raise_error(p.e, DEV_TIMEOUT, 0x440);
            break;
          }
        }
      }
    } else {
      // ================= epilogue warps
      const int ew = warp - C::kEpiWarp0;
      const int quad = warp & 3;         // TMEM lanes this warp may read
      const int grp = ew >> 2;           // decode: tiles n with n % 2 == grp; prefill: token pair
      const int r = quad * 32 + lane;    // key row within the tile
      constexpr int kTokPerWarp = G == 1 ? 1 : 2;
      Cursor<G> cur;
      cur.seek(p, s_seq, s_fseq, n_items);
      int g_seen = 0;                    // query groups whose weights this warp has checked in
      float qs[kTokPerWarp];
      for (int tt = 0; tt < kTokPerWarp; ++tt) qs[tt] = 0.f;
      bool ok = true;
      // fused top-k: this warp's previous candidates, stored once their slot base
      // (an atomic's return) has arrived, so that no tile waits for it
      bool pend_keep = false;
      unsigned pend_mask = 0u;
      int pend_base = 0, pend_s = 0, pend_t = 0;
      float pend_v = 0.f;
      auto flush_pending = [&]() {
        const int pb = __shfl_sync(0xFFFFFFFFu, pend_base, 0);
        if (pend_keep) {
          const long long slot = pb + __popc(pend_mask & ((1u << lane) - 1u));
          if (slot < p.cand_cap) {
            p.cand_score[(long long)pend_t * p.cand_cap + slot] = pend_v;
            p.cand_pos[(long long)pend_t * p.cand_cap + slot] = pend_s;
          }
        }
        pend_keep = false;
      };
      for (long long n = 0; n < n_items; ++n) {
        const int g = cur.gcount - 1;
        const int slot = g & 1;
        const bool mine = G != 1 || (int)(n & 1) == grp;
        if (mine) {
          if (g_seen <= g) {  // first tile of a group for this warp: its weights have landed
            ok = mbar_wait(b_full + slot, (uint32_t)(g >> 1) & 1, p.e, 0x431);
            if (!ok) break;
            g_seen = g + 1;
#pragma unroll
            for (int tt = 0; tt < kTokPerWarp; ++tt) {
              const int t = cur.row0() + (G == 1 ? 0 : grp * 2 + tt);
              qs[tt] = __ldg(p.q_scale + min(t, p.T - 1));
            }
          }
          const int ab = (int)(n % C::kAccBufs);
          const int st = (int)(n % C::kStages);
          ok = mbar_wait(acc_full + ab, (uint32_t)(n / C::kAccBufs) & 1, p.e, 0x430);
          if (!ok) break;
          tc_fence_after();
          const int s = cur.kt * kTileKeys + r;
          const int b = cur.b;
          const bool key_ok = s < cur.s.len;
          float sk = 0.f;
          if (PG || p.scales_bulk) {
            sk = sScale[st * kTileKeys + r];
          } else if (key_ok) {
            if (p.L.page_size == 0) {
              sk = __ldg(p.k_scale + (long long)b * p.L.n_max + s);
            } else {
              const int pg = __ldg(p.L.page_table + (long long)b * p.L.max_pages + s / 64);
              if ((unsigned)pg < (unsigned)p.L.num_pages)
                sk = __ldg(reinterpret_cast<const float *>(p.k_pool + (long long)pg * 8448 + 8192) + (s & 63));
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(a_empty + st);  // keys and scales of this stage are no longer read here
          const int nrows = cur.rows();
          // this warp's accumulator columns: kTokPerWarp tokens x 64 heads, read as
          // 32-column chunks with the next chunk's TMEM load in flight during the math
          constexpr int kCh = kTokPerWarp * 2;
          const int gi0 = G == 1 ? 0 : grp * 2;
          const uint32_t tb = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(ab * C::N + gi0 * kHI);
          uint32_t va[32], vb[32];
          tmem_ld32(tb, va);
          tmem_ld_wait(va);
          float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);  // two packed chains
#pragma unroll
          for (int c = 0; c < kCh; ++c) {
            uint32_t(&cv)[32] = (c & 1) ? vb : va;
            uint32_t(&nv)[32] = (c & 1) ? va : vb;
            if (c + 1 < kCh) tmem_ld32(tb + (uint32_t)((c + 1) * 32), nv);
            const int tt = c >> 1;
            const float4 *w4 = reinterpret_cast<const float4 *>(sW + (slot * G + gi0 + tt) * kHI + (c & 1) * 32);
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const float4 wv = w4[j4];
              const float2 r01 = make_float2(fmaxf(__uint_as_float(cv[4 * j4]), 0.f),
                                             fmaxf(__uint_as_float(cv[4 * j4 + 1]), 0.f));
              const float2 r23 = make_float2(fmaxf(__uint_as_float(cv[4 * j4 + 2]), 0.f),
                                             fmaxf(__uint_as_float(cv[4 * j4 + 3]), 0.f));
              a01 = fma2(make_float2(wv.x, wv.y), r01, a01);
              a23 = fma2(make_float2(wv.z, wv.w), r23, a23);
            }
            if (c & 1) {  // the token's 64 heads are summed: scale and store
              const int gi = gi0 + tt;
              const float acc = (a01.x + a01.y) + (a23.x + a23.y);
              a01 = make_float2(0.f, 0.f);
              a23 = make_float2(0.f, 0.f);
              const long long pos = cur.s.p_first + (long long)cur.i * G + gi;
              const int t = cur.row0() + gi;
              const float v = acc * qs[tt] * sk;
              const bool valid = gi < nrows && key_ok && s <= pos;
              if (G == 1 && F) {
                // the candidates at or above the current bound and their histogram
                // (fire-and-forget atomics), instead of the scores
                const uint32_t bin = order_key(v) >> 20;
                const unsigned long long bp = *reinterpret_cast<volatile unsigned long long *>(&s_bound);
                const unsigned bnd = (int)(bp >> 32) == t ? (unsigned)bp : 0u;
                const bool keep = valid && bin >= bnd;
                if (keep) atomicAdd(p.hist + (long long)t * 4096 + bin, 1u);
                const unsigned mask = __ballot_sync(0xFFFFFFFFu, keep);
                const unsigned wtop = __reduce_max_sync(0xFFFFFFFFu, keep ? bin : 0u);
                if (lane == 0 && mask)  // rows only increase within a CTA: (row, bin) pairs order by max
                  atomicMax(&s_top, ((unsigned long long)(unsigned)t << 32) | wtop);
                flush_pending();
                int base = 0;
                if (lane == 0 && mask) base = atomicAdd(p.cand_count + t, __popc(mask));
                pend_base = base;
                pend_keep = keep;
                pend_mask = mask;
                pend_v = v;
                pend_s = s;
                pend_t = t;
                if (lane == 0 && quad == 0) {
                  *reinterpret_cast<volatile int *>(&s_cur_row) = t;
                  atomicAdd(&s_tiles, 1);
                }
              } else if (valid) {
                p.scores[(long long)t * p.ld + s] = v;
              }
            }
            if (c + 1 < kCh) tmem_ld_wait(nv);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_empty + ab);
        }
        const bool last = n + 1 == n_items;
        const bool newg = cur.next(p);
        if (newg || last) {  // this warp is done with group g: its query slot may be reloaded
          __syncwarp();
          if (lane == 0) mbar_arrive(b_empty + slot);
        }
      }
      if (G == 1 && F) flush_pending();
      __syncwarp();
      if (lane == 0) atomicAdd(&s_epi_done, 1);  // the bound warp stops once all have finished
    }
  }
  if (error_raised(p.e)) {
    // a wait gave up somewhere: copies issued before that may still be in flight
    const unsigned long long t0 = globaltimer();
    while (globaltimer() - t0 < 50000ull) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::kMmaWarp0) tmem_dealloc(tmem, C::kTmemCols);
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

// 2-D byte tensor [rows][128] with 128-byte swizzled boxes of box_rows rows.
bool make_map(CUtensorMap *m, const void *ptr, unsigned long long rows, unsigned box_rows) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int G, bool F, bool PG>
cudaError_t launch_gp(const uint8_t *q, const uint8_t *kI, const Params &p, int num_sms, cudaStream_t stream) {
  using C = Cfg<G>;
  CUtensorMap tq, tk;
  const unsigned long long krows =
      p.L.page_size ? (unsigned long long)p.L.num_pages * 66ull : (unsigned long long)p.L.batch * p.L.n_max;
  if (!make_map(&tq, q, (unsigned long long)p.T * kHI, C::N)) return cudaErrorInvalidValue;
  if (!make_map(&tk, kI, krows, 64)) return cudaErrorInvalidValue;
  cudaError_t err =
      cudaFuncSetAttribute(indexer_fp8_kernel<G, F, PG>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (err != cudaSuccess) return err;
  return launch_kernel(indexer_fp8_kernel<G, F, PG>, dim3(num_sms), dim3(C::kThreads), C::kSmem, stream, 0, tq,
                       tk, p);
}
template <int G, bool F>
cudaError_t launch_g(const uint8_t *q, const uint8_t *kI, const Params &p, int num_sms, cudaStream_t stream) {
  return p.L.page_size ? launch_gp<G, F, true>(q, kI, p, num_sms, stream)
                       : launch_gp<G, F, false>(q, kI, p, num_sms, stream);
}

}  // namespace

int indexer_fp8_grid(int num_sms) { return num_sms; }

cudaError_t launch_indexer_fp8(const uint8_t *q, const float *q_scale, const uint8_t *kI, const float *k_scale,
                               const float *w, int T, const Layout &L, float *scores, long long ld, const ErrCtx &e,
                               int num_sms, cudaStream_t stream) {
  if (L.batch > 8192) return cudaErrorInvalidValue;  // per-sequence prefix lives in stage memory
  Params p;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.k_pool = kI;
  p.w = w;
  p.scores = scores;
  p.scales_bulk = L.page_size != 0 ||
                  ((L.n_max % 4) == 0 && (reinterpret_cast<uintptr_t>(k_scale) & 15u) == 0);
  p.ld = ld;
  p.T = T;
  p.L = L;
  p.e = e;
  p.fuse = 0;
  p.k = 0;
  p.hist = nullptr;
  p.cand_count = nullptr;
  p.cand_score = nullptr;
  p.cand_pos = nullptr;
  p.cand_cap = 0;
  if (L.cu_q == nullptr) return launch_g<1, false>(q, kI, p, num_sms, stream);
  return launch_g<4, false>(q, kI, p, num_sms, stream);
}

namespace {
// Clears the fused top-k's histograms and candidate counts before the indexer
// adds to them (chained by programmatic dependent launch like every kernel here).
__global__ void zero_u32x2_kernel(unsigned *a, long long na, unsigned *b, long long nb) {
  pdl_prologue();
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < na + nb; i += stride) {
    if (i < na) a[i] = 0u;
    else b[i - na] = 0u;
  }
}
}  // namespace

cudaError_t launch_indexer_fp8_fused(const uint8_t *q, const float *q_scale, const uint8_t *kI, const float *k_scale,
                                     const float *w, int T, const Layout &L, int k, unsigned *hist, int *cand_count,
                                     float *cand_score, int *cand_pos, long long cand_cap, const ErrCtx &e,
                                     int num_sms, cudaStream_t stream) {
  if (L.batch > 8192 || L.cu_q != nullptr) return cudaErrorInvalidValue;
  const long long na = (long long)T * 4096, nb = T;
  const int blocks = (int)min((na + nb + 255) / 256, (long long)num_sms * 4);
  cudaError_t err = launch_kernel(zero_u32x2_kernel, dim3(blocks), dim3(256), 0, stream, 0, hist, na,
                                  reinterpret_cast<unsigned *>(cand_count), nb);
  if (err != cudaSuccess) return err;
  Params p;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.k_pool = kI;
  p.w = w;
  p.scores = nullptr;
  p.scales_bulk = L.page_size != 0 ||
                  ((L.n_max % 4) == 0 && (reinterpret_cast<uintptr_t>(k_scale) & 15u) == 0);
  p.ld = 0;
  p.T = T;
  p.L = L;
  p.e = e;
  p.fuse = 1;
  p.k = k;
  p.hist = hist;
  p.cand_count = cand_count;
  p.cand_score = cand_score;
  p.cand_pos = cand_pos;
  p.cand_cap = cand_cap;
  return launch_g<1, true>(q, kI, p, num_sms, stream);
}

}  // namespace dsa
