// Device-side building blocks shared by the DSA kernels (sm_100a only):
// bounded mbarrier waits with a device error word, tcgen05 (TMEM alloc, MMA,
// commit, loads), TMA tile loads, cp.async gathers, UMMA shared-memory and
// instruction descriptors, and the query-row -> (sequence, position) mapping.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a only"
#endif

namespace dsa {

// ---------------------------------------------------------------- error word
// err[0]: OR of the flags below; err[1]: code of the first failing site.
enum : unsigned { DEV_TIMEOUT = 1u, DEV_BOUNDS = 2u };

struct ErrCtx {
  unsigned *word;            // device pointer to two unsigned ints
  unsigned long long limit;  // wait bound in ns
};

__device__ __forceinline__ void raise_error(const ErrCtx &e, unsigned flag, unsigned site) {
  unsigned old = atomicOr(e.word, flag);
  if (old == 0) atomicExch(e.word + 1, site);
}

// True once any wait has timed out: the remaining waits then give up at once.
__device__ __forceinline__ bool error_raised(const ErrCtx &e) {
  return (*(volatile unsigned *)e.word & DEV_TIMEOUT) != 0;
}

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// As above, but the thread may sleep up to `hint_ns` waiting for the phase,
// instead of polling: waiting warps then leave the issue slots to working ones.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Slow path of mbar_wait: sleeping waits, each at most 1 ms (and at most the
// limit), until the phase
// completes, another wait has timed out, or the deadline passes (DEV_TIMEOUT
// recorded with `site`).
static __device__ __noinline__ bool mbar_wait_slow(uint64_t *bar, uint32_t parity, const ErrCtx &e, unsigned site) {
  const unsigned long long t0 = globaltimer();
  const uint32_t hint = (uint32_t)(e.limit < 1000000ull ? e.limit : 1000000ull);  // never sleep past the limit
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, hint)) return true;
    if (error_raised(e)) return false;
    if (globaltimer() - t0 > e.limit) {
      raise_error(e, DEV_TIMEOUT, site);
      return false;
    }
  }
}

// Waits for the phase with the given parity to complete. Returns false (after
// recording DEV_TIMEOUT with `site`) when the wait exceeds the limit, or at once
// when another wait has already timed out, so that every role can wind down.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, const ErrCtx &e, unsigned site) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, e, site);
}

// Waits (bounded) until the shared counter *c equals `target` (a turn counter
// that orders work handed out to several warps).
__device__ __forceinline__ bool wait_turn(const volatile int *c, int target, const ErrCtx &e, unsigned site) {
  if (*c == target) return true;
  const unsigned long long t0 = globaltimer();
  while (*c != target) {
    __nanosleep(64);
    if (error_raised(e)) return false;
    if (globaltimer() - t0 > e.limit) {
      raise_error(e, DEV_TIMEOUT, site);
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------- proxies / fences
// Programmatic dependent launch (kernels launched with programmatic stream
// serialization): the next kernel on the stream may be scheduled once every CTA
// of this one has called pdl_launch_dependents(); pdl_wait() returns once the
// previous kernel has completed and its writes are visible. Every kernel here
// calls both first thing, so completion stays ordered kernel by kernel.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_prologue() {
  pdl_wait();
  pdl_launch_dependents();
}

// Bring a global line toward L2 ahead of its first use (no register result).
__device__ __forceinline__ void prefetch_l2(const void *ptr) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---------------------------------------------------------------- packed fp32
// {a.x, a.y} += {w.x, w.y} * {x.x, x.y} as one packed fp32x2 FMA (round to nearest)
__device__ __forceinline__ float2 fma2(float2 w, float2 x, float2 a) {
  unsigned long long wv, xv, av, d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(wv) : "f"(w.x), "f"(w.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(xv) : "f"(x.x), "f"(x.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(av) : "f"(a.x), "f"(a.y));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(wv), "l"(xv), "l"(av));
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
  return r;
}

// ---------------------------------------------------------------- TMEM
// Allocation and deallocation are warp-wide (.sync.aligned).
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// columns [col, col+32) of TMEM lane (lane base of the address) + i.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Waits for this thread's TMEM loads and makes `r` (the destination of the last
// one) an operand of the wait, so no use of it can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]),
        "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]),
        "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
        "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread i of the warp writes r[0..15]
// into columns [col, col+16) of TMEM lane (lane base of the address) + i.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- UMMA
// Shared-memory matrix descriptor (tcgen05): start address, leading and stride
// byte offsets (16-byte units), version 1, swizzle mode in bits [61,64).
enum : uint32_t { SW_NONE = 0, SW_128B = 2 };

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t swizzle) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)(swizzle & 7) << 61;
  return d;
}

// Instruction descriptor for dense kind::f16 / kind::f8f6f4 with fp32 accumulate.
// a_fmt/b_fmt: kind::f16 -> 0 f16, 1 bf16; kind::f8f6f4 -> 0 e4m3.
// a_mn/b_mn: 0 = K-major operand, 1 = MN-major operand.
__host__ __device__ constexpr uint32_t instr_desc(uint32_t a_fmt, uint32_t b_fmt, uint32_t a_mn, uint32_t b_mn,
                                                  uint32_t M, uint32_t N) {
  return (1u << 4)            // D format: f32
         | (a_fmt << 7) | (b_fmt << 10) | (a_mn << 15) | (b_mn << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// As umma_f16 with the A operand in TMEM: M rows in lanes 0..M-1, the K values of
// a row packed two 16-bit values per 32-bit column (the lower K index in the low half).
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives once on `bar` when every MMA issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------- TMA / bulk / cp.async
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
// Four rows y0..y3 of a 2-D tensor map whose box is one row high: columns x .. x+box-1
// of each row land as four consecutive box rows at dst (swizzled like a tiled load);
// a row outside the tensor is filled with zeros. Completes on `bar` with 4 x box bytes.
__device__ __forceinline__ void tma_gather4(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y0, int y1,
                                            int y2, int y3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3)
      : "memory");
}
// Plain (untiled) bulk copy global -> shared, completing on `bar` with tx bytes.
// Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Plain bulk copy shared -> global in this thread's bulk async-group. Both
// addresses 16-byte aligned, size a multiple of 16; the shared-memory source must
// have been made visible to the async proxy (fence_proxy_async_smem) first.
__device__ __forceinline__ void bulk_store(void *dst, const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until every bulk async-group of this thread has finished reading its
// shared-memory source (the writes may still be in flight; they complete with the grid).
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void *src, bool valid) {
  const uint32_t n = valid ? 16u : 0u;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
// The barrier counts this thread's arrival once all its earlier cp.async copies land.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Byte offset of 16-byte chunk `c` (0..7) of row `r` in a 128-byte-swizzled tile
// whose rows are 128 bytes and whose base is 1024-byte aligned.
__host__ __device__ __forceinline__ uint32_t sw128_off(uint32_t r, uint32_t c) {
  return r * 128u + ((c ^ (r & 7u)) << 4);
}

// ---------------------------------------------------------------- rows
struct Layout {
  int row0;  // query row t of a launch is row (row0 + t) of the caller's rows
  int batch;
  const int *seq_lens;
  const int *cu_q;
  int page_size;
  const int *page_table;
  int max_pages;
  int num_pages;
  int n_max;
};

struct RowPos {
  int b;    // sequence
  int pos;  // position of the query token
  int len;  // keys in the sequence
};

// Query row t -> (sequence, position). Decode: row t is sequence t's newest
// token. Prefill: binary search of t in cu_q.
__device__ __forceinline__ RowPos row_position(const Layout &L, int t) {
  RowPos r;
  t += L.row0;
  if (L.cu_q == nullptr) {
    r.b = t;
    r.len = __ldg(L.seq_lens + t);
    r.pos = r.len - 1;
  } else {
    int lo = 0, hi = L.batch;  // find b with cu_q[b] <= t < cu_q[b+1]
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (__ldg(L.cu_q + mid) <= t) lo = mid; else hi = mid;
    }
    r.b = lo;
    r.len = __ldg(L.seq_lens + lo);
    const int q0 = __ldg(L.cu_q + lo), q1 = __ldg(L.cu_q + lo + 1);
    r.pos = r.len - (q1 - q0) + (t - q0);
  }
  return r;
}

// Largest number of keys a sequence may hold under this layout.
__device__ __forceinline__ int cache_capacity(const Layout &L) {
  return L.page_size ? L.max_pages * L.page_size : L.n_max;
}

// Physical row of key s of sequence b (contiguous: b*n_max + s; paged: page*P + slot),
// or -1 (with DEV_BOUNDS recorded) when the page id is out of range.
__device__ __forceinline__ long long key_row(const Layout &L, int b, int s, const ErrCtx &e, unsigned site) {
  if (L.page_size == 0) return (long long)b * L.n_max + s;
  const int page = __ldg(L.page_table + (long long)b * L.max_pages + s / L.page_size);
  if ((unsigned)page >= (unsigned)L.num_pages) {
    raise_error(e, DEV_BOUNDS, site);
    return -1;
  }
  return (long long)page * L.page_size + (s % L.page_size);
}

}  // namespace dsa
