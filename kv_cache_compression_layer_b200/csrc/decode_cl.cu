// kv_decode_attn_update on bf16 caches with g <= 8 query heads per KV head,
// for batches whose rows fill the GPU as clusters (rows x C about the SM
// count): one decode step (VoxZip, second stage: A^(t) = gamma [A^(t-1), 0]
// + softmax(q_t K_t^T / sqrt d), then keep the T sinks, the M most recent
// entries and the top-N of the middle by A) with every row one thread-block
// cluster of C CTAs, so that nothing about a row leaves the cluster.
//
// CTA c of a row's cluster owns slots [c S, min((c+1) S, b+1)), S the row's
// b + 1 slots over the C CTAs rounded up to whole 64-slot tiles. Its twelve
// warps (three groups of four, each group streaming its own 64-slot tiles of
// K and V by TMA through two stages) run the tensor-core online softmax of
// the persistent kernel (decode_tc.cu). Every logit goes to tensor memory
// (the lane and columns of the thread that computed it), not to global
// memory. At the end the groups' (max, sum, O) are combined in shared
// memory, the cluster's CTAs combine theirs through distributed shared
// memory (log-denominators per query head, the attention output split over
// the CTAs), each warp reads its logits back from tensor memory to add the
// exact probabilities into A for its slots, and cluster rank 0 picks the
// eviction from the CTAs' candidates and writes the row's meta data. The
// only waits are the groups' bounded TMA waits and hardware cluster barriers.
#include <cooperative_groups.h>

#include "decode_tc_common.cuh"

namespace cg = cooperative_groups;

namespace kvc {
namespace {

struct ClArgs {
  DecArgs a;
  int C;         // CTAs per row (cluster size)
  int S;         // slots per CTA (a multiple of 64)
  int cpg;       // tensor-memory columns per group (a multiple of 32): 4 per tile of the group
  int ncols;     // tensor-memory columns per CTA (a power of two >= 3 cpg)
  unsigned long long limit_ns;
};

// The row's step state, the same for every CTA of the row.
struct ClRow {
  long long base;
  int cap, count, next, steps, count0, bb, n, pos_new, pos_thr, ok, evict, lo, hi, ntiles;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) decode_cl_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                const __grid_constant__ CUtensorMap tmV,
                                                                const __grid_constant__ CUtensorMap tmQ,
                                                                const __grid_constant__ ClArgs P) {
  constexpr int NDC = D / 16;
  constexpr int TILE = kTcSlots * D * 2;
  constexpr int STAGE = 2 * TILE + kQBytes;
  const DecArgs& a = P.a;
  const int G = a.G, E = G * D;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = warp >> 2, gt = tid & 127, wq = warp & 3;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / P.C;

  extern __shared__ uint8_t dsm_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  float* o_s = reinterpret_cast<float*>(ring + kStages * STAGE);  // [groups][G][D], swizzled columns
  __shared__ uint64_t full[kStages];
  __shared__ int st0_s[kStages];          // first slot of the tile in a stage (-1: the group is done)
  __shared__ float red_m[kWarps][kTcMaxG], red_l[kWarps][kTcMaxG];
  __shared__ float gm[kGroups][kTcMaxG], gl[kGroups][kTcMaxG];  // the groups' (max, sum)
  __shared__ float cm[kTcMaxG], cl[kTcMaxG];                    // this CTA's (max, sum): read by rank 0
  __shared__ float fM[kTcMaxG], fLi[kTcMaxG], flse[kTcMaxG];    // the row's, written by rank 0
  __shared__ Best wbest[kWarps];
  __shared__ Best cbest;                                         // this CTA's candidate: read by rank 0
  __shared__ ClRow R;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s, nreal_s[kGroups], more_s[kGroups];

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&full[i], 1);
    abort_s = 0;
    fence_barrier_init();
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmQ);
  }
  if (warp == 0) {
    tmem_alloc(&tmem_s, (uint32_t)P.ncols);
    tmem_relinquish();
  }
  for (int i = tid; i < kGroups * G * D; i += kThreads) o_s[i] = 0.f;
  pdl_wait();  // the previous step has finished with the cache
  pdl_launch_dependents();
  if (tid == 0) {
    const int32_t* meta = a.meta + (long long)row * 8;
    R.count = meta[0];
    R.next = meta[1];
    R.steps = meta[2];
    R.count0 = meta[4];
    R.base = a.slot_off[row];
    R.cap = (int)(a.slot_off[row + 1] - R.base);
    R.bb = a.b[row];
    R.n = R.count + 1;
    const int Mr = (a.recent_pct * R.bb) / 100;
    const int appended = R.steps + 1;
    R.evict = R.n > R.bb;
    R.ok = R.count < R.cap && R.next >= 0 && R.next < R.cap && (!R.evict || R.bb >= a.T + Mr);
    R.pos_new = row_len(a.map, row) + R.steps;
    R.pos_thr = R.pos_new - Mr + 1;
    if (R.ok && appended < Mr) R.pos_thr = a.pos[R.base + max(0, R.count0 - (Mr - appended))];
    // the row's slots split evenly over the cluster in whole tiles (P.S bounds the share)
    const int share = ((R.cap + P.C - 1) / P.C + kTcSlots - 1) / kTcSlots * kTcSlots;
    R.lo = min(rank * share, R.cap);
    R.hi = min(R.lo + share, R.cap);
    R.ntiles = (R.hi - R.lo + kTcSlots - 1) / kTcSlots;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  const Guard gd{&abort_s, a.status, P.limit_ns};
  const int lo = R.lo, hi = R.hi, ntiles = R.ntiles;
  const long long base = R.base;

  // ---------------------------------------------------------------- attention
  // group grp takes the CTA's tiles grp, grp + 3, ...; tile t covers slots [lo + 64 t, ...)
  if (gt == 0) {
    const uint64_t policy = make_policy_evict_first();
    int n_real = 0;
    bool ended = false;
    for (int s = 0; s < kGStages && !ended; ++s) {
      const int stg = grp * kGStages + s;
      const int t = grp + kGroups * n_real;
      if (t < ntiles) {
        st0_s[stg] = lo + t * kTcSlots;
        mbar_arrive_expect_tx(&full[stg], 2 * TILE + G * D * 2);
        const int y = (int)(base + lo + t * kTcSlots);
        uint8_t* stage = ring + stg * STAGE;
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx) {
          tma_load_2d_hint(stage + bx * kTcSlots * 128, &tmK, &full[stg], bx * 64, y, policy);
          tma_load_2d_hint(stage + TILE + bx * kTcSlots * 128, &tmV, &full[stg], bx * 64, y, policy);
          tma_load_2d(stage + 2 * TILE + bx * 1024, &tmQ, &full[stg], bx * 64, row * G);
        }
        ++n_real;
      } else {
        st0_s[stg] = -1;
        mbar_arrive(&full[stg]);
        ended = true;
      }
    }
    nreal_s[grp] = n_real;
    more_s[grp] = !ended;
  }

  const int g0 = lane >> 2, q4 = lane & 3;
  const bool g_ok = g0 < G;
  const int m_ = lane >> 3, r_ = lane & 7;
  const int wslot = wq * 16;  // this warp's 16 slots of a tile
  const bool row_ok = R.ok != 0;
  const int n = R.n, next = R.next;
  float* og = o_s + grp * G * D;
  bool aborted = false;
  float m0 = -INFINITY, l0 = 0.f;
  float o[2 * NDC][2];
#pragma unroll
  for (int i = 0; i < 2 * NDC; ++i) o[i][0] = o[i][1] = 0.f;
  int k = 0;
  for (;; ++k) {
    const int stg = grp * kGStages + (k & 1);
    // the group decides together whether the stage arrived (its warps' barriers
    // and warp-wide instructions must not part)
    const bool got = named_bar_and(1 + grp, 128, !aborted && wait_bounded(&full[stg], (k >> 1) & 1, gd));
    if (!got) aborted = true;
    const int st0 = got ? st0_s[stg] : -1;
    if (st0 < 0) break;
    const int t = grp + kGroups * k;  // the tile's index in this CTA
    uint8_t* stage = ring + stg * STAGE;
    const uint32_t ktile = smem_u32(stage), vtile = ktile + TILE;
    if (row_ok && next >= st0 + wslot && next < st0 + wslot + 16 && next < hi) {
      // the appended token: patch its K and V rows into the tile, write them to the cache
      const int r = next - st0;
      const __nv_bfloat16* kin = static_cast<const __nv_bfloat16*>(a.k) + (long long)row * D;
      const __nv_bfloat16* vin = static_cast<const __nv_bfloat16*>(a.v) + (long long)row * D;
      if (lane < D / 8) {
        const uint4 kv = *reinterpret_cast<const uint4*>(kin + lane * 8);
        const uint4 vv = *reinterpret_cast<const uint4*>(vin + lane * 8);
        *reinterpret_cast<uint4*>(stage + (swz(ktile, r, lane * 8) - ktile)) = kv;
        *reinterpret_cast<uint4*>(stage + (swz(vtile, r, lane * 8) - ktile)) = vv;
        reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.Kc) + (base + next) * D)[lane] = kv;
        reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.Vc) + (base + next) * D)[lane] = vv;
      }
      if (lane == 0) a.pos[base + next] = R.pos_new;
      fence_proxy_async();
      __syncwarp();
    }
    // logits S = Q K^T for this warp's 16 slots (two n-tiles of 8 slots, even and
    // odd d-chunks in separate accumulators)
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t qarea = ktile + 2 * TILE;
    const int qrow = (lane & 7) < G ? (lane & 7) : 0;  // rows >= G are zeroed below
#pragma unroll
    for (int dc = 0; dc < NDC; ++dc) {
      uint32_t b00, b01, b10, b11, qa0, qa1;
      ldsm_x2(qswz(qarea, qrow, dc * 16 + ((lane >> 3) & 1) * 8), qa0, qa1);
      ldsm_x4(swz(ktile, wslot + (m_ >> 1) * 8 + r_, dc * 16 + (m_ & 1) * 8), b00, b01, b10, b11);
      const uint32_t af[4] = {g_ok ? qa0 : 0u, 0u, g_ok ? qa1 : 0u, 0u};
      if (dc & 1) {
        mma16816(t0, af, b00, b01);
        mma16816(t1, af, b10, b11);
      } else {
        mma16816(s0, af, b00, b01);
        mma16816(s1, af, b10, b11);
      }
    }
    const int jb = st0 + wslot + q4 * 2;  // slots jb, jb+1 (n-tile 0) and jb+8, jb+9 (n-tile 1)
    float x[4];
    x[0] = s0[0] + t0[0];
    x[1] = s0[1] + t0[1];
    x[2] = s1[0] + t1[0];
    x[3] = s1[1] + t1[1];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = jb + (e & 1) + (e >> 1) * 8;
      const bool valid = row_ok && j < n && j < hi;
      x[e] = valid ? x[e] * a.scale2 : -INFINITY;
    }
    // the logits stay on chip: this thread's lane, the group's columns 4 k .. 4 k + 3
    tmem_st4(tmem + ((uint32_t)(wq * 32) << 16) + grp * P.cpg + 4 * k, x[0], x[1], x[2], x[3]);
    // online softmax update of this warp's running (max, sum, O)
    float tm = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 1));
    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 2));
    const float nm = fmaxf(m0, tm);
    const float vm = nm == -INFINITY ? 0.f : nm;
    if (__any_sync(0xffffffffu, nm != m0)) {
      const float sc0 = ex2_approx(m0 - vm);
      l0 *= sc0;
#pragma unroll
      for (int i = 0; i < 2 * NDC; ++i) {
        o[i][0] *= sc0;
        o[i][1] *= sc0;
      }
    }
    m0 = nm;
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      p[e] = ex2_approx(x[e] - vm);
      l0 += p[e];
    }
    const uint32_t pa[4] = {pack_bf16(p[0], p[1]), 0u, pack_bf16(p[2], p[3]), 0u};
#pragma unroll
    for (int dn = 0; dn < NDC; ++dn) {
      uint32_t b0a, b1a, b0b, b1b;
      ldsm_x4_t(swz(vtile, wslot + (m_ & 1) * 8 + r_, dn * 16 + (m_ >> 1) * 8), b0a, b1a, b0b, b1b);
      float c0[4] = {o[2 * dn][0], o[2 * dn][1], 0.f, 0.f};
      float c1[4] = {o[2 * dn + 1][0], o[2 * dn + 1][1], 0.f, 0.f};
      mma16816(c0, pa, b0a, b1a);
      mma16816(c1, pa, b0b, b1b);
      o[2 * dn][0] = c0[0];
      o[2 * dn][1] = c0[1];
      o[2 * dn + 1][0] = c1[0];
      o[2 * dn + 1][1] = c1[1];
    }
    named_bar_sync(1 + grp, 128);  // the group is done with this stage: refill it
    if (gt == 0 && more_s[grp]) {
      const int tn = grp + kGroups * nreal_s[grp];
      if (tn < ntiles) {
        st0_s[stg] = lo + tn * kTcSlots;
        mbar_arrive_expect_tx(&full[stg], 2 * TILE + G * D * 2);
        const int y = (int)(base + lo + tn * kTcSlots);
        const uint64_t policy = make_policy_evict_first();
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx) {
          tma_load_2d_hint(stage + bx * kTcSlots * 128, &tmK, &full[stg], bx * 64, y, policy);
          tma_load_2d_hint(stage + TILE + bx * kTcSlots * 128, &tmV, &full[stg], bx * 64, y, policy);
          tma_load_2d(stage + 2 * TILE + bx * 1024, &tmQ, &full[stg], bx * 64, row * G);
        }
        ++nreal_s[grp];
      } else {
        st0_s[stg] = -1;
        mbar_arrive(&full[stg]);
        more_s[grp] = 0;
      }
    }
  }
  if (aborted) {
    abort_s = 1;
    if (gt == 0)  // let this group's copies in flight land before the CTA goes on
      for (int tt = k; tt < nreal_s[grp]; ++tt)
        wait_drain(&full[grp * kGStages + (tt & 1)], (tt >> 1) & 1);
  }
  // the group's running (max, sum, O): warps combined into (gm, gl) and og
  {
    float ls0 = l0;
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) ls0 += __shfl_xor_sync(0xffffffffu, ls0, off);
    if (q4 == 0 && g_ok) {
      red_m[warp][g0] = m0;
      red_l[warp][g0] = ls0;
    }
    named_bar_sync(1 + grp, 128);
    float M0 = -INFINITY;
    if (g_ok)
      for (int w4 = 0; w4 < 4; ++w4) M0 = fmaxf(M0, red_m[grp * 4 + w4][g0]);
    const float f0 = m0 == -INFINITY ? 0.f : ex2_approx(m0 - M0);
    // the group's warps add their O in warp order (a fixed summation order, so
    // a step's result does not depend on scheduling); lanes own distinct columns
#pragma unroll
    for (int w4 = 0; w4 < 4; ++w4) {
      if (wq == w4 && g_ok) {
#pragma unroll
        for (int i = 0; i < 2 * NDC; ++i) {
          const int col = i * 8 + q4 * 2;
          og[g0 * D + ogswz(g0, col)] += o[i][0] * f0;
          og[g0 * D + ogswz(g0, col + 1)] += o[i][1] * f0;
        }
      }
      if (w4 < 3) named_bar_sync(1 + grp, 128);
    }
    if (gt < G) {
      float M = -INFINITY;
      for (int w4 = 0; w4 < 4; ++w4) M = fmaxf(M, red_m[grp * 4 + w4][gt]);
      float Ls = 0.f;
      for (int w4 = 0; w4 < 4; ++w4)
        if (red_m[grp * 4 + w4][gt] > -INFINITY)
          Ls += red_l[grp * 4 + w4][gt] * ex2_approx(red_m[grp * 4 + w4][gt] - M);
      gm[grp][gt] = M;
      gl[grp][gt] = Ls;
    }
  }
  tc_wait_st();  // this thread's logits are in tensor memory
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ------------------------------------------------------------------ finish
  const bool skip = abort_s || (*reinterpret_cast<volatile int32_t*>(a.status) & KV_DEV_TIMEOUT) != 0;
  float* o_cta = reinterpret_cast<float*>(ring);            // [G][D] this CTA's O (the ring is free now)
  float* A_s = o_cta + kTcMaxG * D;                          // [S] A of this CTA's slots
  int* pos_s = reinterpret_cast<int*>(A_s + P.S);            // [S] their positions
  float* wr = reinterpret_cast<float*>(pos_s + P.S);         // [C][G] weights of the CTAs' partials
  // (1) this CTA's slot data for the sweep (copied while the partials are combined)
  for (int i = tid; i < hi - lo; i += kThreads) {
    cp_async4(A_s + i, a.A + base + lo + i);
    cp_async4(pos_s + i, a.pos + base + lo + i);
  }
  // this CTA's (max, sum, O) from its three groups
  if (tid < G) {
    float M = -INFINITY;
    for (int g2 = 0; g2 < kGroups; ++g2) M = fmaxf(M, gm[g2][tid]);
    float L = 0.f;
    for (int g2 = 0; g2 < kGroups; ++g2)
      if (gm[g2][tid] > -INFINITY) L += gl[g2][tid] * ex2_approx(gm[g2][tid] - M);
    cm[tid] = M;
    cl[tid] = L;
  }
  __syncthreads();
  for (int i = tid; i < E; i += kThreads) {
    const int g = i / D, c = i % D;
    float v = 0.f;
    for (int g2 = 0; g2 < kGroups; ++g2)
      if (gm[g2][g] > -INFINITY) v += o_s[(g2 * G + g) * D + ogswz(g, c)] * ex2_approx(gm[g2][g] - cm[g]);
    o_cta[i] = v;
  }
  cluster.sync();  // every CTA's (max, sum, O) is ready

  // (2) the row's log-denominators per query head, by rank 0 into every CTA
  if (rank == 0 && tid < G) {
    float M = -INFINITY;
    for (int r = 0; r < P.C; ++r) M = fmaxf(M, cluster.map_shared_rank(cm, r)[tid]);
    float L = 0.f;
    for (int r = 0; r < P.C; ++r) {
      const float mr = cluster.map_shared_rank(cm, r)[tid];
      if (mr > -INFINITY) L += cluster.map_shared_rank(cl, r)[tid] * ex2_approx(mr - M);
    }
    for (int r = 0; r < P.C; ++r) {
      cluster.map_shared_rank(fM, r)[tid] = M;
      cluster.map_shared_rank(fLi, r)[tid] = L > 0.f ? 1.f / L : 0.f;
      cluster.map_shared_rank(flse, r)[tid] = M + log2f(L);
    }
  }
  cluster.sync();
  if (tid < P.C * G) {  // weight of CTA r's partial for head g
    const int r = tid / G, g = tid % G;
    const float mr = cluster.map_shared_rank(cm, r)[g];
    wr[tid] = mr > -INFINITY ? ex2_approx(mr - fM[g]) : 0.f;
  }
  cp_async_wait_all();
  __syncthreads();

  // (3) this CTA's share of the row's attention output
  {
    const int e0 = (int)((long long)E * rank / P.C), e1 = (int)((long long)E * (rank + 1) / P.C);
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + (long long)row * E;
    for (int i = e0 + tid; i < e1; i += kThreads) {
      const int g = i / D;
      float v = 0.f;
      for (int r = 0; r < P.C; ++r) v += cluster.map_shared_rank(o_cta, r)[i] * wr[r * G + g];
      if (!skip) out[i] = __float2bfloat16_rn(v * fLi[g]);
    }
  }

  // (4) decayed scores of this warp's own slots from its logits in tensor memory
  Best best{INFINITY, -1, -1};
  {
    const float lse_g = g_ok ? flse[g0] : 0.f;
    const bool upd = !skip && row_ok;
    const int nk = ntiles > grp ? (ntiles - grp + kGroups - 1) / kGroups : 0;  // this group's tiles
    for (int k0 = 0; k0 < nk; k0 += 8) {
      float xs[32];  // eight tiles' logits in one load
      tmem_ld32(tmem + ((uint32_t)(wq * 32) << 16) + grp * P.cpg + 4 * k0, xs);
      tc_wait_ld();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
      if (k0 + kk >= nk) break;
      const int t = grp + kGroups * (k0 + kk);
      float ps[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) ps[e] = g_ok ? ex2_approx(xs[4 * kk + e] - lse_g) : 0.f;
#pragma unroll
      for (int off = 4; off < 32; off <<= 1)  // sum over the query heads (lanes with the same q4)
#pragma unroll
        for (int e = 0; e < 4; ++e) ps[e] += __shfl_xor_sync(0xffffffffu, ps[e], off);
      if (g0 == 0 && upd) {
        const int jb = lo + t * kTcSlots + wslot + q4 * 2;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = jb + (e & 1) + (e >> 1) * 8;
          if (j < n && j < hi) {
            const float Anew = (j == next ? 0.f : a.gamma * A_s[j - lo]) + ps[e];
            a.A[base + j] = Anew;
            const int pj = j == next ? R.pos_new : pos_s[j - lo];
            if (j >= a.T && pj < R.pos_thr) {
              const Best c{Anew, pj, j};
              if (better(c, best)) best = c;
            }
          }
        }
      }
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    Best y;
    y.A = __shfl_xor_sync(0xffffffffu, best.A, off);
    y.pos = __shfl_xor_sync(0xffffffffu, best.pos, off);
    y.slot = __shfl_xor_sync(0xffffffffu, best.slot, off);
    if (better(y, best)) best = y;
  }
  if (lane == 0) wbest[warp] = best;
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    Best b = wbest[0];
    for (int w = 1; w < kWarps; ++w)
      if (better(wbest[w], b)) b = wbest[w];
    cbest = b;
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, (uint32_t)P.ncols);
  }
  cluster.sync();  // every CTA's candidate is ready

  // (5) the eviction and the row's meta data, by rank 0
  if (rank == 0 && tid == 0) {
    Best b{INFINITY, -1, -1};
    for (int r = 0; r < P.C; ++r) {
      const Best c = *cluster.map_shared_rank(&cbest, r);
      if (better(c, b)) b = c;
    }
    int32_t* meta = a.meta + (long long)row * 8;
    if (!row_ok) {
      atomicOr(a.status, KV_DEV_BUDGET);
    } else if (!skip) {
      if (R.evict && b.slot >= 0) {
        meta[0] = R.bb;
        meta[1] = b.slot;
        meta[3] = b.slot;
      } else {
        meta[0] = R.n;
        meta[1] = R.n;
        meta[3] = -1;
      }
      meta[2] = R.steps + 1;
    }
  }
  cluster.sync();  // rank 0 has read the other CTAs' shared memory
}

}  // namespace

// A batch takes this path when its rows fill the GPU as clusters of C <= 8
// CTAs (C a power of two, rows x C between 7/8 of the SM count and the SM
// count) and a CTA's share of the largest row fits its tensor memory.
int cl_cluster_size(const kv_shape& sh, const RowMap& m, int capb) {
  const int sms = sm_count();
  for (int C = 8; C >= 1; C >>= 1) {
    const long long ctas = (long long)m.n_rows * C;
    if (ctas > sms || ctas * 8 < (long long)sms * 7) continue;
    const int S = ((capb + C - 1) / C + kTcSlots - 1) / kTcSlots * kTcSlots;
    const int cpg = (4 * ((S / kTcSlots + kGroups - 1) / kGroups) + 31) / 32 * 32;
    if (kGroups * cpg > 512) return 0;
    // shared memory of the finish: O, A and positions of S slots, the CTAs' weights
    const size_t fin = (size_t)kTcMaxG * sh.head_dim * 4 + (size_t)S * 8 + 8 * kTcMaxG * 4;
    const size_t ring = (size_t)kStages * (2 * kTcSlots * sh.head_dim * 2 + kQBytes);
    if (fin > ring) return 0;
    return C;
  }
  return 0;
}

int launch_cl(const kv_shape& sh, const RowMap& m, int capb, int C, long long total_slots, const DecArgs& a,
              const kv_cache& c, cudaStream_t st) {
  if (total_slots >= (1ll << 31)) return KV_ERR_ARG;
  ClArgs P;
  P.a = a;
  P.C = C;
  P.S = ((capb + C - 1) / C + kTcSlots - 1) / kTcSlots * kTcSlots;
  P.cpg = (4 * ((P.S / kTcSlots + kGroups - 1) / kGroups) + 31) / 32 * 32;
  int cols = 32;
  while (cols < kGroups * P.cpg) cols <<= 1;
  P.ncols = cols;
  P.limit_ns = wait_limit_ns();
  const int stage_bytes = 2 * kTcSlots * sh.head_dim * 2 + kQBytes;
  const size_t smem = 1024 + (size_t)kStages * stage_bytes + (size_t)kGroups * sh.group * sh.head_dim * 4;
  CUtensorMap tmK, tmV, tmQ;
  if (!encode_rows_bf16(&tmK, c.Kc, sh.head_dim, total_slots, kTcSlots)) return KV_ERR_CUDA;
  if (!encode_rows_bf16(&tmV, c.Vc, sh.head_dim, total_slots, kTcSlots)) return KV_ERR_CUDA;
  if (!encode_rows_bf16(&tmQ, a.q, sh.head_dim, (long long)m.n_rows * sh.group, sh.group)) return KV_ERR_CUDA;
  auto kern = sh.head_dim == 128 ? decode_cl_kernel<128> : decode_cl_kernel<64>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return KV_ERR_ARG;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // the launch may start while the previous step's kernel drains (programmatic
  // dependent launch); it waits (griddepcontrol.wait) before touching memory
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(m.n_rows * C);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, tmK, tmV, tmQ, P));
}

}  // namespace kvc
