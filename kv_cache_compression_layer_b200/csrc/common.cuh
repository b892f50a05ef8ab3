// Shared device helpers for the sm_100a kernels: row/tile maps of a ragged
// batch, mbarrier waits with a time limit, TMA tile loads, and the tcgen05
// (5th-generation tensor core + tensor memory) instructions used by scoring.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvcomp.h"

namespace kvc {

constexpr int kTileKeys = 128;  // keys per scoring tile (the MMA's M or N)

// Index checks of debug builds. kv_check(ok) returns ok; when it is false it
// sets KV_DEV_BOUNDS in this file's check word, and the caller skips the
// access. Each kernel file has its own word (a device variable is local to
// its file without relocatable device code) and registers a reader with the
// C-ABI layer, which ORs them. Release builds compile kv_check to `true`.
#ifdef KV_DEBUG_CHECKS
constexpr bool kDebugChecks = true;
namespace {
__device__ int kv_check_word_;
int read_check_word(bool clear) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, kv_check_word_, sizeof(int)) != cudaSuccess) return -1;
  if (clear) {
    const int z = 0;
    if (cudaMemcpyToSymbol(kv_check_word_, &z, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}
}  // namespace
void register_check_word(int (*reader)(bool));
namespace {
struct CheckWordRegistration {
  CheckWordRegistration() { register_check_word(&read_check_word); }
} check_word_registration_;
}  // namespace
__device__ __forceinline__ bool kv_check(bool ok) {
  if (!ok) atomicOr(&kv_check_word_, KV_DEV_BOUNDS);
  return ok;
}
#else
constexpr bool kDebugChecks = false;
__device__ __forceinline__ bool kv_check(bool) { return true; }
#endif

// Where every row of a ragged batch lives. Rows of sequence s are
// rows_per_seq consecutive rows of length L[s].
struct RowMap {
  int n_seq;
  int rows_per_seq;  // n_layers * n_kv_heads
  int n_rows;
  int L[KV_MAX_SEQ];
  long long key_off[KV_MAX_SEQ + 1];  // first key of sequence s
  int tile_off[KV_MAX_SEQ + 1];       // first scoring tile of sequence s
};

__device__ __forceinline__ int row_seq(const RowMap& m, int row) { return row / m.rows_per_seq; }
__device__ __forceinline__ int row_len(const RowMap& m, int row) { return m.L[row / m.rows_per_seq]; }
__device__ __forceinline__ long long row_key_off(const RowMap& m, int row) {
  int s = row / m.rows_per_seq;
  return m.key_off[s] + (long long)(row - s * m.rows_per_seq) * m.L[s];
}
// Scoring tile u -> (row, tile within the row).
__device__ __forceinline__ void tile_to_row(const RowMap& m, int u, int& row, int& tile) {
  int s = 0;
  while (s + 1 < m.n_seq && m.tile_off[s + 1] <= u) ++s;
  int tpr = (m.L[s] + kTileKeys - 1) / kTileKeys;
  int local = u - m.tile_off[s];
  row = s * m.rows_per_seq + local / tpr;
  tile = local % tpr;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{.reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0];}" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{.reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;}" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{.reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p;}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}

// Non-blocking test of a phase.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{.reg .pred p; mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p;}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: gives up once `abort` is raised by another thread of the CTA,
// or after limit_ns of its own, in which case it raises `abort` and records
// KV_DEV_TIMEOUT in the device status word. Returns false when it gave up.
// A limit of 0 gives up on any wait whose phase has not completed already
// (no suspended try), which lets a test drive every kernel's timeout path.
struct Guard {
  volatile int* abort;  // shared-memory flag of the CTA
  int* status;          // device status word
  unsigned long long limit_ns;
};

__device__ __forceinline__ bool give_up(const Guard& g) {
  *g.abort = 1;
  atomicOr(g.status, KV_DEV_TIMEOUT);
  return false;
}

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, const Guard& g) {
  if (g.limit_ns == 0) return mbar_test_wait(bar, parity) ? true : give_up(g);
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*g.abort) return false;
    if (globaltimer() - t0 > g.limit_ns) return give_up(g);
  }
}

// Wait used while draining after an abort (copies or MMAs already issued
// must land before the CTA releases its shared or tensor memory): ignores the
// abort flag and has a limit of its own, independent of the waits' limit.
constexpr unsigned long long kDrainLimitNs = 2000000000ull;
__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity) {
  uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > kDrainLimitNs) return false;
  }
}

// Named barrier over `nthreads` threads that also ANDs a predicate across them:
// every participant gets the same result.
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{.reg .pred p, q; setp.ne.u32 p, %3, 0; bar.red.and.pred q, %1, %2, p; selp.u32 %0, 1, 0, q;}"
      : "=r"(r)
      : "r"(id), "r"(nthreads), "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

// The bin of the kk-th largest key from a 256-bin histogram, by one warp: lane
// l holds bins 255 - 8 l down to 248 - 8 l, so lanes in order walk the bins
// from the top. Returns the bin; kk becomes the rank within it. The bins must
// hold at least kk keys in all.
__device__ __forceinline__ int top_bin(const int* hist, int& kk) {
  const int lane = threadIdx.x & 31;
  int loc[8], tot = 0;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    loc[t] = hist[255 - 8 * lane - t];
    tot += loc[t];
  }
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int excl = incl - tot;
  const unsigned here = __ballot_sync(0xffffffffu, excl < kk && kk <= incl);
  const int src = __ffs(here) - 1;
  int dg = 0, kk_new = kk;
  if (lane == src) {
    int cum = excl;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (cum + loc[t] >= kk) {
        dg = 255 - 8 * lane - t;
        kk_new = kk - cum;
        break;
      }
      cum += loc[t];
    }
  }
  dg = __shfl_sync(0xffffffffu, dg, src);
  kk = __shfl_sync(0xffffffffu, kk_new, src);
  return dg;
}

// ---------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
// Same, with an L2 cache-eviction policy (from make_policy_*).
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t make_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t make_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void st_f32_hint(float* addr, float v, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(addr), "f"(v), "l"(policy) : "memory");
}
// The same store without a compiler memory clobber, so values already loaded
// stay in registers across it: callers order it against later reads of the
// same data with a barrier or fence.
__device__ __forceinline__ void st_f32_hint_nc(float* addr, float v, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(addr), "f"(v), "l"(policy));
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{.reg .pred p; setp.ne.b32 p, %4, 0;"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on an mbarrier once every previously issued tcgen05.mma has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// The same wait, with the 32 registers a tcgen05.ld filled as operands, so no
// use of them can be scheduled before it.
__device__ __forceinline__ void tc_wait_ld_regs(float (&v)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]), "+f"(v[7]),
                 "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]), "+f"(v[12]), "+f"(v[13]), "+f"(v[14]),
                 "+f"(v[15]), "+f"(v[16]), "+f"(v[17]), "+f"(v[18]), "+f"(v[19]), "+f"(v[20]), "+f"(v[21]),
                 "+f"(v[22]), "+f"(v[23]), "+f"(v[24]), "+f"(v[25]), "+f"(v[26]), "+f"(v[27]), "+f"(v[28]),
                 "+f"(v[29]), "+f"(v[30]), "+f"(v[31])
               :
               : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Shared-memory matrix descriptor of a K-major operand stored in 128-byte
// swizzled rows (8-row groups 1024 bytes apart), as TMA writes it with
// CU_TENSOR_MAP_SWIZZLE_128B. Fields: start address >> 4 (bits 0-13),
// leading byte offset >> 4 (16-29, unused for swizzled K-major), stride byte
// offset >> 4 (32-45), descriptor version 1 (46-47), swizzle mode 2 = 128B
// (61-63).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B, fp32 D, both K-major:
// D format (bits 4-5) = 1 (f32), A format (7-9) = 1 (bf16), B format
// (10-12) = 1 (bf16), N >> 3 (17-22), M >> 4 (24-28).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Arrive at a named barrier without waiting (the producer side of a hand-off).
__device__ __forceinline__ void named_bar_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start its
// set-up now / wait until the previous kernel has finished and its writes are visible.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ bool elect_lane0() { return (threadIdx.x & 31) == 0; }

}  // namespace kvc
