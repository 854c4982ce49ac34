// Fine-grained token selection: per query row, the k best indexer scores over
// the row's causal prefix (jdon.com "DeepSeek-V3.2-Exp", sparse-training and
// selection paragraphs: K = 2048 tokens kept per query; openi.cn "DeepSeek-V3.2",
// token-selection item).
//
// One thread-block cluster of C CTAs per row. Each CTA holds a contiguous
// slice of the row in shared memory as order-preserving 32-bit keys, and the
// cluster runs a 4-pass, 8-bit radix select of the k-th largest key with the
// per-pass histograms summed over distributed shared memory. Selected
// positions are then written in ascending position order: key > threshold, plus
// the lowest-position ties at the threshold. The HBM row is read exactly once.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

// Monotone map float -> uint32: larger float, larger key; -0 and +0 share a key;
// every NaN maps below -inf.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Shared {
  unsigned hist[2][256];
  unsigned total[256];
  unsigned warp_gt[kWarps], warp_eq[kWarps];
  unsigned cta_cnt[2];  // (greater, equal) counts of this CTA, read by the peers
  unsigned prefix, mask, krem;
  unsigned out_base, eq_take;
};

__global__ void __launch_bounds__(kThreads) topk_kernel(const float *__restrict__ scores, long long ld, int k,
                                                        Layout L, int cap, int *__restrict__ idx, ErrCtx e) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Shared &sm = *reinterpret_cast<Shared *>(smem_raw);
  uint32_t *keys = reinterpret_cast<uint32_t *>(smem_raw + ((sizeof(Shared) + 15) & ~size_t(15)));

  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int t = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

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

  // ---- this CTA's slice of the row, as keys in shared memory
  const int chunk = (int)((((n + C - 1) / C) + 31) / 32 * 32);
  const long long lo = (long long)rank * chunk;
  const int cnt = (int)max(0LL, min(n, lo + chunk) - lo);
  const float *row = scores + (long long)t * ld + lo;
  {
    const int n4 = cnt >> 2;
    const float4 *r4 = reinterpret_cast<const float4 *>(row);
    for (int i = tid; i < n4; i += kThreads) {
      float4 v = __ldcs(r4 + i);
      uint4 kk = make_uint4(order_key(v.x), order_key(v.y), order_key(v.z), order_key(v.w));
      reinterpret_cast<uint4 *>(keys)[i] = kk;
    }
    for (int i = (n4 << 2) + tid; i < cnt; i += kThreads) keys[i] = order_key(__ldcs(row + i));
  }
  if (tid == 0) {
    sm.prefix = 0;
    sm.mask = 0;
    sm.krem = (unsigned)k;
  }

  // contiguous per-warp segments (multiples of 32) keep lanes converged
  const int seg = ((cnt + kWarps * 32 - 1) / (kWarps * 32)) * 32;
  const int wlo = warp * seg;

  // ---- radix select of the k-th largest key, 8 bits per pass
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    unsigned *h = sm.hist[pass & 1];
    for (int i = tid; i < 256; i += kThreads) h[i] = 0;
    __syncthreads();
    const unsigned prefix = sm.prefix, mask = sm.mask;
    for (int j = lane; j < seg; j += 32) {
      const int i = wlo + j;
      int bin = -1;
      if (i < cnt) {
        const uint32_t key = keys[i];
        if ((key & mask) == prefix) bin = (int)((key >> shift) & 255u);
      }
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, bin);
      if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&h[bin], (unsigned)__popc(peers));
    }
    cluster.sync();
    if (tid < 256) {
      unsigned s = 0;
      for (int r = 0; r < C; ++r) s += cluster.map_shared_rank(h, r)[tid];
      sm.total[tid] = s;
    }
    __syncthreads();
    if (warp == 0) {
      const unsigned krem = sm.krem;
      unsigned v[8], s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[i] = sm.total[lane * 8 + i];
        s += v[i];
      }
      unsigned suf = s;  // inclusive suffix sum over lanes
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned o = __shfl_down_sync(0xFFFFFFFFu, suf, off);
        if (lane + off < 32) suf += o;
      }
      const unsigned above = suf - s;
      if (above < krem && krem <= suf) {
        unsigned c = above;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          if (c + v[i] >= krem) {
            sm.prefix = prefix | ((unsigned)(lane * 8 + i) << shift);
            sm.mask = mask | (255u << shift);
            sm.krem = krem - c;
            break;
          }
          c += v[i];
        }
      }
    }
    __syncthreads();
  }
  const uint32_t thr = sm.prefix;
  const unsigned krem = sm.krem;  // ties at the threshold still to take

  // ---- counts per warp, per CTA, then across the cluster
  {
    unsigned gt = 0, eq = 0;
    for (int j = lane; j < seg; j += 32) {
      const int i = wlo + j;
      const uint32_t key = i < cnt ? keys[i] : 0u;
      const bool in = i < cnt;
      gt += __popc(__ballot_sync(0xFFFFFFFFu, in && key > thr));
      eq += __popc(__ballot_sync(0xFFFFFFFFu, in && key == thr));
    }
    if (lane == 0) {
      sm.warp_gt[warp] = gt;
      sm.warp_eq[warp] = eq;
    }
  }
  __syncthreads();
  if (tid == 0) {
    unsigned g = 0, q = 0;
    for (int w = 0; w < kWarps; ++w) {
      const unsigned a = sm.warp_gt[w], b = sm.warp_eq[w];
      sm.warp_gt[w] = g;  // exclusive prefixes
      sm.warp_eq[w] = q;
      g += a;
      q += b;
    }
    sm.cta_cnt[0] = g;
    sm.cta_cnt[1] = q;
  }
  cluster.sync();
  if (tid == 0) {
    unsigned gt_before = 0, eq_before = 0;
    for (int r = 0; r < rank; ++r) {
      const unsigned *pc = cluster.map_shared_rank(sm.cta_cnt, r);
      gt_before += pc[0];
      eq_before += pc[1];
    }
    const unsigned mine = sm.cta_cnt[1];
    const unsigned taken_before = min(eq_before, krem);
    sm.eq_take = min(mine, krem - taken_before);
    sm.out_base = gt_before + taken_before;
  }
  cluster.sync();  // peers are done reading this CTA's counts after this point

  // ---- emit selected positions in ascending order
  {
    const unsigned eq_take = sm.eq_take;
    const unsigned eq_pre = sm.warp_eq[warp];
    unsigned base = sm.out_base + sm.warp_gt[warp] + min(eq_pre, eq_take);
    unsigned tie = eq_pre;
    const unsigned lt = (1u << lane) - 1u;
    for (int j = lane; j < seg; j += 32) {
      const int i = wlo + j;
      const bool in = i < cnt;
      const uint32_t key = in ? keys[i] : 0u;
      const bool is_eq = in && key == thr;
      const unsigned eqm = __ballot_sync(0xFFFFFFFFu, is_eq);
      const bool take = (in && key > thr) || (is_eq && tie + __popc(eqm & lt) < eq_take);
      const unsigned selm = __ballot_sync(0xFFFFFFFFu, take);
      if (take) {
        const unsigned p = base + __popc(selm & lt);
        if (p < (unsigned)k) out[p] = (int)(lo + i);
      }
      base += __popc(selm);
      tie += __popc(eqm);
    }
  }
}

}  // namespace

size_t topk_smem_bytes(int cap) { return ((sizeof(Shared) + 15) & ~size_t(15)) + (size_t)cap * 4; }

cudaError_t launch_topk(const float *scores, long long ld, int T, int k, const Layout &L, int C, int cap, int *idx,
                        const ErrCtx &e, cudaStream_t stream) {
  const size_t smem = topk_smem_bytes(cap);
  cudaError_t err = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  if (C > 8) {
    err = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return err;
  }
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
  return cudaLaunchKernelEx(&cfg, topk_kernel, scores, ld, k, L, cap, idx, e);
}

}  // namespace dsa
