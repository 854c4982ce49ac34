// Fine-grained token selection: per query row, the k best indexer scores over
// the row's causal prefix (jdon.com "DeepSeek-V3.2-Exp", sparse-training and
// selection paragraphs: K = 2048 tokens kept per query; openi.cn "DeepSeek-V3.2",
// token-selection item).
//
// One thread-block cluster of C CTAs per row. Each CTA holds a contiguous slice
// of the row in shared memory as order-preserving 32-bit keys. The cluster finds
// the key of the k-th best score by radix select in three passes (11, 11 and 10
// bits; the first histogram is built while loading), summing the per-CTA
// histograms over distributed shared memory. Selected positions are then written
// in ascending order: keys above the threshold plus the lowest-position keys equal
// to it. The row is read from HBM exactly once.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins1 = 2048, kBins2 = 2048, kBins3 = 1024;  // bits 31..21, 20..10, 9..0

// Monotone map float -> uint32: larger float, larger key; -0 and +0 share a key;
// every NaN maps below -inf.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Shared {
  unsigned hist1[kBins1], hist2[kBins2], hist3[kBins3];
  unsigned wsum[kWarps];
  unsigned wsum2[kWarps];
  unsigned cta_cnt[2];  // (greater, equal) counts of this CTA, read by the peers
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

// Sum over the cluster of W consecutive bins per thread (all peers read at once).
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
    } else {
      const uint2 q = *reinterpret_cast<const uint2 *>(ph);
      peer[r][0] = q.x;
      peer[r][1 % W] = q.y;
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
  for (int i = tid; i < kBins2; i += kThreads) sm.hist2[i] = 0;
  for (int i = tid; i < kBins3; i += kThreads) sm.hist3[i] = 0;
  __syncthreads();

  // ---- this CTA's slice as keys in shared memory; histogram of bits 31..21
  const int chunk = (int)((((n + C - 1) / C) + 31) / 32 * 32);
  const long long lo = (long long)rank * chunk;
  const int cnt = (int)max(0LL, min(n, lo + chunk) - lo);
  {
    const float *row = scores + (long long)t * ld + lo;
    const int n4 = cnt >> 2;
    const float4 *r4 = reinterpret_cast<const float4 *>(row);
    constexpr int U = 8;  // float4 loads in flight per thread
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
          atomicAdd(sm.hist1 + (kk.x >> 21), 1u);
          atomicAdd(sm.hist1 + (kk.y >> 21), 1u);
          atomicAdd(sm.hist1 + (kk.z >> 21), 1u);
          atomicAdd(sm.hist1 + (kk.w >> 21), 1u);
        }
      }
    }
    const int i = (n4 << 2) + tid;  // 0..3 trailing keys
    if (i < cnt) {
      const uint32_t kx = order_key(__ldcs(row + i));
      keys[i] = kx;
      atomicAdd(sm.hist1 + (kx >> 21), 1u);
    }
  }

  // ---- pass 1: bits 31..21
  cluster.sync();
  unsigned krem = (unsigned)k;
  uint32_t prefix;
  {
    unsigned v[4];
    cluster_counts<C, 4>(cluster, sm.hist1, v);
    find_bin<4>(v, krem, sm);
    prefix = sm.sel_bin;  // top 11 bits
    krem = sm.sel_krem;
  }
  // ---- pass 2: bits 20..10 among keys whose top 11 bits match
#pragma unroll 4
  for (int i = tid; i < cnt; i += kThreads) {
    const uint32_t key = keys[i];
    if ((key >> 21) == prefix) atomicAdd(sm.hist2 + ((key >> 10) & 2047u), 1u);
  }
  cluster.sync();
  {
    unsigned v[4];
    cluster_counts<C, 4>(cluster, sm.hist2, v);
    find_bin<4>(v, krem, sm);
    prefix = (prefix << 11) | sm.sel_bin;  // top 22 bits
    krem = sm.sel_krem;
  }
  // ---- pass 3: bits 9..0 among keys whose top 22 bits match
#pragma unroll 4
  for (int i = tid; i < cnt; i += kThreads) {
    const uint32_t key = keys[i];
    if ((key >> 10) == prefix) atomicAdd(sm.hist3 + (key & 1023u), 1u);
  }
  cluster.sync();
  {
    unsigned v[2];
    cluster_counts<C, 2>(cluster, sm.hist3, v);
    find_bin<2>(v, krem, sm);
    prefix = (prefix << 10) | sm.sel_bin;  // the threshold key
    krem = sm.sel_krem;                    // keys equal to it still to take
  }
  const uint32_t thr = prefix;

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
    unsigned gt_before = 0, eq_before = 0;
#pragma unroll
    for (int r = 0; r < C; ++r)
      if (r < rank) {
        gt_before += pc[r][0];
        eq_before += pc[r][1];
      }
    const unsigned taken_before = min(eq_before, krem);
    sm.eq_take = min(cta_eq, krem - taken_before);
    sm.out_base = gt_before + taken_before;
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)T * C);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_kernel<C>, scores, ld, k, L, cap, idx, e);
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
