// kv_decode_attn_update on bf16 caches with g <= 8 query heads per KV head:
// one persistent launch per decode step (VoxZip, second stage:
// A^(t) = gamma [A^(t-1), 0] + softmax(q_t K_t^T / sqrt d), then keep the T
// sinks, the M most recent entries and the top-N of the middle by A).
//
// Every row's b + 1 slots are cut into work items of kCH slots; one CTA per
// SM takes a contiguous run of items, so each CTA owns a contiguous range of
// the slot space. The runs are cut at equal shares of a cost that counts the
// slots and charges each row once more (a row costs its groups a combine of
// their running softmax state and a partial written out), so CTAs holding
// many short rows get fewer slots.
//
// Attention phase. Twelve warps form three groups of four. The CTA's items
// are cut into three contiguous runs, one per group, walked as 64-slot tiles
// (a row change then costs one group, not all three, a combine); a group
// claims its run's items one at a time from the front, and a group that has
// run out takes the back half of the largest unclaimed run of another group
// (a shared (front, back) word per group, changed by compare-and-swap), so
// the groups of a CTA end together. Each group feeds itself: its first thread streams its
// tiles (K and V as 128-byte swizzled TMA boxes, the row's g query rows as a
// bulk copy, a header with the row's step state) into the group's two
// stages, and refills a stage as soon as the group has finished with it.
// In a group each warp owns 16 slots of a tile and runs one pass of online
// softmax on the tensor cores (mma.sync m16n8k16: A = the g query rows padded
// to 16, B = K rows via ldmatrix; then A = P, B = V rows via ldmatrix.trans).
// Every logit goes to an L2-resident scratch; when a group leaves a row it
// combines its four warps into one (max, sum, O) partial and lists it for
// the row. The appended token's K and V rows are patched into the tile that
// holds its slot and written to the cache by the warp that owns that slot.
//
// Grid barrier (all CTAs are resident: one per SM by shared memory; the
// wait is bounded and reports KV_DEV_TIMEOUT).
//
// Finish phase. (1) Output units of 256 elements of a row's g x d output,
// spread over every warp of the grid, combine the row's partials into the
// attention output. (2) Each CTA computes the row constants (log2 of the
// softmax denominators per query head, eviction thresholds) of the rows in
// its range; then every warp sweeps its share of the CTA's slots, adds the
// exact probabilities into A and proposes its smallest middle A per row
// piece. The piece that completes a row's slot count picks the eviction
// from the row's proposals and writes the row's meta data for the next step.
#include "decode_tc_common.cuh"

namespace kvc {
namespace {

// Scratch of the tensor-core path inside kv_cache.scratch.
struct TcScratch {
  int* n_items;    // [1]
  int* item_off;   // [rows + 1] first item of each row
  int2* items;     // [max_items] (row, chunk)
  float* part;     // [max_items * kGroups][stride]: max[G] at 0, sum[G] at G, O[G][d] at kPartO,
                   // per (first item of a group's segment, group)
  float* logits;   // [total_slots][8] logits in log2 units (heads >= G hold -inf)
  int* plist;      // [rows][max_per_row * kGroups] list entries (PEnt: per-head max and sum, index,
                   // step stamp), one place per (item that starts a group's segment, group)
  int* done;       // [rows] slots of the row finished in the current step
  int* best_n;     // [rows] eviction proposals of the row in the current step
  int4* bests;     // [rows][max_bests] proposals (A bits, pos, slot, -)
  unsigned* attn_done;  // [rows] slots of the row attended so far (grows by the row's capacity
                        // every step; the decode init clears it)
  long long* row_cost;  // [rows + 1] prefix of the rows' costs (slots + kRowCost)
  int* cta_u;           // [kMaxCtas + 1] first item of each CTA's run; cta_u[kMaxCtas] = the grid it was cut for
  int max_items, max_per_row, stride, max_bests;
};

// The cost of a row beyond its slots when cutting the CTAs' runs, in slots: a
// row change makes a group combine its four warps' softmax state and write a
// partial, during which its stages wait, and adds a row's statistics and
// output to the CTA's finish (measured together: about what 150 slots take).
constexpr int kRowCost = 150;
constexpr int kMaxCtas = 1024;

struct TcArgs {
  DecArgs a;
  TcScratch sc;
  unsigned long long limit_ns;
};

// What a group's first thread learns about a tile and hands to its group.
struct TileHdr {
  int row, u, st0, c1, count, next, steps, cap;  // row = -1: the group's tiles are done
  long long base;
};

size_t tc_layout(int rows, int G, int d, int capb, long long total_slots, char* base, TcScratch* sc) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int per_row = (capb + kCH - 1) / kCH;
  // rows hold at most per_row items each and sum(b + 1) = total_slots slots in all
  const int max_items = (int)std::min<long long>((long long)rows * per_row, total_slots / kCH + rows);
  const int stride = (kPartO + G * d + 3) & ~3;
  const int max_bests = (per_row + 1) * kWarps;
  size_t off = 0;
  const size_t o_n = off;
  off += 256;
  const size_t o_ioff = off;
  off += al((size_t)(rows + 1) * 4);
  const size_t o_items = off;
  off += al((size_t)max_items * 8);
  const size_t o_part = off;
  off += al((size_t)max_items * kGroups * stride * 4);
  const size_t o_log = off;
  off += al((size_t)total_slots * kTcMaxG * 4);
  const size_t o_pl = off;
  off += al((size_t)rows * per_row * kGroups * 80);
  const size_t o_done = off;
  off += al((size_t)rows * 4);
  const size_t o_bn = off;
  off += al((size_t)rows * 4);
  const size_t o_best = off;
  off += al((size_t)rows * max_bests * 16);
  const size_t o_ad = off;
  off += al((size_t)rows * 4);
  const size_t o_rc = off;
  off += al((size_t)(rows + 1) * 8);
  const size_t o_cu = off;
  off += al((size_t)(kMaxCtas + 1) * 4);
  if (sc && base) {
    sc->n_items = reinterpret_cast<int*>(base + o_n);
    sc->item_off = reinterpret_cast<int*>(base + o_ioff);
    sc->items = reinterpret_cast<int2*>(base + o_items);
    sc->part = reinterpret_cast<float*>(base + o_part);
    sc->logits = reinterpret_cast<float*>(base + o_log);
    sc->plist = reinterpret_cast<int*>(base + o_pl);
    sc->done = reinterpret_cast<int*>(base + o_done);
    sc->best_n = reinterpret_cast<int*>(base + o_bn);
    sc->bests = reinterpret_cast<int4*>(base + o_best);
    sc->attn_done = reinterpret_cast<unsigned*>(base + o_ad);
    sc->row_cost = reinterpret_cast<long long*>(base + o_rc);
    sc->cta_u = reinterpret_cast<int*>(base + o_cu);
    sc->max_items = max_items;
    sc->max_per_row = per_row;
    sc->stride = stride;
    sc->max_bests = max_bests;
  }
  return off;
}

// Builds the work items of every row (rows cut into kCH-slot chunks), clears
// the per-row step counters, and cuts the items into n_cta runs of equal cost
// (slots + kRowCost per row); one block.
__global__ void tc_items_kernel(int n_rows, const int64_t* __restrict__ slot_off, TcScratch sc, int n_cta,
                                int32_t* __restrict__ status) {
  __shared__ int warp_tot[32];
  __shared__ long long warp_cost[32];
  __shared__ int carry;
  __shared__ long long carry_cost;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    carry = 0;
    carry_cost = 0;
  }
  __syncthreads();
  for (int base = 0; base < n_rows; base += blockDim.x) {
    const int i = base + threadIdx.x;
    int own = 0;
    long long cost = 0;
    if (i < n_rows) {
      const long long cap = slot_off[i + 1] - slot_off[i];
      own = (int)((cap + kCH - 1) / kCH);
      if (own > sc.max_per_row) {
        atomicOr(status, KV_DEV_CAPACITY);
        own = sc.max_per_row;
      }
      cost = cap + kRowCost;
    }
    int v = own;
    long long vc = cost;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      const long long yc = __shfl_up_sync(0xffffffffu, vc, o);
      if (lane >= o) {
        v += y;
        vc += yc;
      }
    }
    if (lane == 31) {
      warp_tot[warp] = v;
      warp_cost[warp] = vc;
    }
    __syncthreads();
    int wb = 0;
    long long wbc = 0;
    for (int k = 0; k < warp; ++k) {
      wb += warp_tot[k];
      wbc += warp_cost[k];
    }
    const int incl = carry + wb + v;
    const long long incl_c = carry_cost + wbc + vc;
    if (i < n_rows) {
      sc.done[i] = 0;
      sc.best_n[i] = 0;
      sc.attn_done[i] = 0;
      sc.item_off[i] = incl - own;
      sc.row_cost[i] = incl_c - cost;
      for (int c = 0; c < own; ++c) sc.items[incl - own + c] = make_int2(i, c);
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) {
      carry = incl;
      carry_cost = incl_c;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    sc.item_off[n_rows] = carry;
    sc.row_cost[n_rows] = carry_cost;
    *sc.n_items = carry;
  }
  __syncthreads();
  // CTA b starts at the first item whose cost prefix reaches total * b / n_cta:
  // item c of row i starts at P_i (c = 0) or P_i + kRowCost + c kCH (c >= 1)
  const long long total = carry_cost;
  const int n_items = carry;
  for (int i = threadIdx.x; i < n_rows; i += blockDim.x) {
    const long long P0 = sc.row_cost[i], P1 = sc.row_cost[i + 1];
    const int own = sc.item_off[i + 1] - sc.item_off[i];
    // the boundaries b with P0 < total * b / n_cta <= P1
    int b = (int)((P0 * n_cta) / total);
    while ((total * b) / n_cta <= P0) ++b;
    for (; b < n_cta && (total * b) / n_cta <= P1; ++b) {
      const long long T = (total * b) / n_cta;
      long long c = (T - P0 - kRowCost + kCH - 1) / kCH;
      if (c < 1) c = 1;
      sc.cta_u[b] = c < own ? sc.item_off[i] + (int)c : sc.item_off[i] + own;
    }
  }
  if (threadIdx.x == 0) {
    sc.cta_u[0] = 0;
    sc.cta_u[n_cta] = n_items;
    sc.cta_u[kMaxCtas] = n_cta;
  }
}

// The walk over a CTA's tiles in issue order (items u0..u1 in turn, each cut
// into 64-slot tiles). A group's first thread keeps one; the next row's
// state is loaded one row ahead so that a row change does not stall it.
struct Walk {
  int u, u1;           // current item, end of the CTA's items
  int t, nt;           // tile within the item, tiles of the item
  int it;              // CTA-wide index of the current tile
  int row, chunk, nchunk, c1;
  int cap, count, next, steps;
  long long base;
  long long nend;      // slot_off[row + 2]
  int ncount, nnext, nsteps;
};

__device__ __forceinline__ void walk_prefetch(Walk& w, const DecArgs& a, int max_per_row) {
  w.nchunk = min((w.cap + kCH - 1) / kCH, max_per_row);
  if (w.row + 1 < a.map.n_rows) {  // next row's state, consumed at the next row change
    w.nend = a.slot_off[w.row + 2];
    const int32_t* m = a.meta + (long long)(w.row + 1) * 8;
    w.ncount = m[0];
    w.nnext = m[1];
    w.nsteps = m[2];
  }
}

__device__ __forceinline__ void walk_item(Walk& w) {
  const int c0 = w.chunk * kCH;
  w.c1 = min(c0 + kCH, w.cap);
  w.nt = (w.c1 - c0 + kTcSlots - 1) / kTcSlots;
  w.t = 0;
}

// Positions the walk on tile 0 of the CTA; false when the CTA has no items.
__device__ __forceinline__ bool walk_first(Walk& w, const DecArgs& a, const TcScratch& sc, int u0, int u1) {
  w.u = u0;
  w.u1 = u1;
  w.it = 0;
  if (u0 >= u1) return false;
  const int2 item = sc.items[u0];
  w.row = item.x;
  w.chunk = item.y;
  w.base = a.slot_off[w.row];
  w.cap = (int)(a.slot_off[w.row + 1] - w.base);
  const int32_t* m = a.meta + (long long)w.row * 8;
  w.count = m[0];
  w.next = m[1];
  w.steps = m[2];
  walk_prefetch(w, a, sc.max_per_row);
  walk_item(w);
  return true;
}

// A group's unclaimed items [front, back) in one 64-bit word: the group
// claims from the front, other groups steal from the back.
__device__ __forceinline__ unsigned long long pack_range(int f, int b) {
  return (unsigned long long)(unsigned)f | ((unsigned long long)(unsigned)b << 32);
}
__device__ __forceinline__ int range_front(unsigned long long c) { return (int)(unsigned)(c & 0xffffffffull); }
__device__ __forceinline__ int range_back(unsigned long long c) { return (int)(unsigned)(c >> 32); }

// Claims item u, the front of the group's range, unless it has been stolen.
__device__ __forceinline__ bool claim_item(unsigned long long* own, int u) {
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(own);
  for (;;) {
    if (range_front(cur) != u || u >= range_back(cur)) return false;
    const unsigned long long prev = atomicCAS(own, cur, pack_range(u + 1, range_back(cur)));
    if (prev == cur) return true;
    cur = prev;
  }
}

// Takes the back half of the largest unclaimed range of another group (at
// least two items left there); false when no group has that much left.
__device__ __forceinline__ bool steal_range(unsigned long long* owns, int grp, int& s0, int& s1) {
  for (;;) {
    int v = -1, best = 1;
    unsigned long long cv = 0;
    for (int g = 0; g < kGroups; ++g) {
      if (g == grp) continue;
      const unsigned long long c = *reinterpret_cast<volatile unsigned long long*>(owns + g);
      const int rem = range_back(c) - range_front(c);
      if (rem > best) {
        best = rem;
        v = g;
        cv = c;
      }
    }
    if (v < 0) return false;
    const int f = range_front(cv), b = range_back(cv), k = (b - f) / 2;
    if (atomicCAS(owns + v, cv, pack_range(f, b - k)) == cv) {
      s0 = b - k;
      s1 = b;
      return true;
    }
  }
}

// Positions the walk on the next item the group may take: the front of its
// own range, else the first of a range stolen from another group (which
// becomes its own). False when the CTA has no unclaimed item worth taking.
__device__ __noinline__ bool group_take(Walk& w, const DecArgs& a, const TcScratch& sc, unsigned long long* owns,
                                        int grp) {
  for (;;) {
    const unsigned long long c = *reinterpret_cast<volatile unsigned long long*>(owns + grp);
    const int f = range_front(c);
    if (claim_item(owns + grp, f)) return walk_first(w, a, sc, f, range_back(c));
    int s0, s1;
    if (!steal_range(owns, grp, s0, s1)) return false;
    atomicExch(owns + grp, pack_range(s0, s1));
  }
}

// Moves to the next tile of the group's claimed items; false when the next
// item cannot be claimed (the range is used up or its rest was stolen).
__device__ __forceinline__ bool walk_advance(Walk& w, const DecArgs& a, int max_per_row, unsigned long long* own) {
  ++w.it;
  if (++w.t < w.nt) return true;
  if (!claim_item(own, w.u + 1)) return false;
  ++w.u;
  if (++w.chunk >= w.nchunk) {  // the next row
    w.chunk = 0;
    w.base += w.cap;
    w.cap = (int)(w.nend - w.base);
    w.count = w.ncount;
    w.next = w.nnext;
    w.steps = w.nsteps;
    ++w.row;
    walk_prefetch(w, a, max_per_row);
  }
  walk_item(w);
  return true;
}


// Streams the walk's current tile into a stage: header, K and V boxes, query rows.
template <int D>
__device__ __forceinline__ void issue_tile(const Walk& w, uint8_t* stage, uint64_t* bar, TileHdr* h,
                                           const CUtensorMap* tmK, const CUtensorMap* tmV, const CUtensorMap* tmQ,
                                           const DecArgs& a, uint64_t policy) {
  constexpr int TILE = kTcSlots * D * 2;
  const int q_bytes = a.G * D * 2;
  h->row = w.row;
  h->u = w.u;
  h->st0 = w.chunk * kCH + w.t * kTcSlots;
  h->c1 = w.c1;
  h->count = w.count;
  h->next = w.next;
  h->steps = w.steps;
  h->cap = w.cap;
  h->base = w.base;
  mbar_arrive_expect_tx(bar, 2 * TILE + q_bytes);
  const int y = (int)(w.base + h->st0);
#pragma unroll
  for (int bx = 0; bx < D / 64; ++bx) {
    tma_load_2d_hint(stage + bx * kTcSlots * 128, tmK, bar, bx * 64, y, policy);
    tma_load_2d_hint(stage + TILE + bx * kTcSlots * 128, tmV, bar, bx * 64, y, policy);
  }
#pragma unroll
  for (int bx = 0; bx < D / 64; ++bx) tma_load_2d(stage + 2 * TILE + bx * 1024, tmQ, bar, bx * 64, w.row * a.G);
}

// One entry of a row's partial list: the partial's per-head (max, sum) and index.
struct PEnt {
  float m[kTcMaxG];
  float l[kTcMaxG];
  int pidx, stamp, pad1, pad2;  // stamp: the row's step number + 1 when written
};
static_assert(sizeof(PEnt) == 80, "list entry layout");

__device__ __forceinline__ void ld_pent(const PEnt* e, float (&m)[kTcMaxG], float (&l)[kTcMaxG], int& pidx,
                                        int& stamp) {
  const float4* v = reinterpret_cast<const float4*>(e);
  const float4 a0 = __ldcg(v), a1 = __ldcg(v + 1), b0 = __ldcg(v + 2), b1 = __ldcg(v + 3);
  const int2 ps = __ldcg(reinterpret_cast<const int2*>(v + 4));
  pidx = ps.x;
  stamp = ps.y;
  m[0] = a0.x; m[1] = a0.y; m[2] = a0.z; m[3] = a0.w; m[4] = a1.x; m[5] = a1.y; m[6] = a1.z; m[7] = a1.w;
  l[0] = b0.x; l[1] = b0.y; l[2] = b0.z; l[3] = b0.w; l[4] = b1.x; l[5] = b1.y; l[6] = b1.z; l[7] = b1.w;
}

// A row's softmax statistics for the finish (in the freed tile ring).
constexpr int kStatParts = 64;  // partials of a row held on chip by the finish (more: read again)
struct RowStat {
  int pidx[kStatParts];              // the row's first partials' indices
  float pm[kStatParts][kTcMaxG];     // their maxima
  float M[kTcMaxG], Li[kTcMaxG], lse[kTcMaxG];
  int nr;                      // partials listed (capped at the list size)
};

// Constants of one row for the finish.
struct RowC {
  long long base;
  unsigned target;  // attended-slot count at which every CTA has finished the row's attention
  int cap, n, next, pos_new, pos_thr, bb, steps, flags;  // flags: 1 ok, 2 evict, 4 too many partials
};

// The row's softmax statistics per query head, merged by one warp from the
// partials this step listed for the row: the list has a place per (item,
// group) of the row's ncand places, and the places written this step carry
// the step's stamp. M_g, 1/L_g and lse_g = M_g + log2 L_g go to ws with the
// first kStatParts partials' indices and maxima (ws.nr = all partials found).
// The entries carry each partial's (max, sum): one round of loads.
__device__ __forceinline__ void row_stats(const TcArgs& P, int row, int ncand, int stamp, int lane, RowStat& ws) {
  const DecArgs& a = P.a;
  const TcScratch& sc = P.sc;
  const int G = a.G;
  const int maxp = sc.max_per_row * kGroups;
  const PEnt* lst = reinterpret_cast<const PEnt*>(sc.plist) + (long long)row * maxp;
  ncand = min(ncand, maxp);
  float m[kTcMaxG], l[kTcMaxG];
#pragma unroll
  for (int g = 0; g < kTcMaxG; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
  }
  int found = 0;  // partials found so far (warp-uniform)
  constexpr int kPer = 3;  // places per lane per round, all loads in flight together
  for (int k0 = 0; k0 < ncand; k0 += 32 * kPer) {
    float em[kPer][kTcMaxG], el[kPer][kTcMaxG];
    int ep[kPer], es[kPer];
#pragma unroll
    for (int h = 0; h < kPer; ++h) {
      es[h] = 0;
      ep[h] = 0;
      const int k = k0 + h * 32 + lane;
      if (k < ncand) ld_pent(lst + k, em[h], el[h], ep[h], es[h]);
    }
#pragma unroll
    for (int h = 0; h < kPer; ++h) {
      const bool valid = k0 + h * 32 + lane < ncand && es[h] == stamp;
      const unsigned bal = __ballot_sync(0xffffffffu, valid);
      const int idx = found + __popc(bal & ((1u << lane) - 1));
      found += __popc(bal);
      if (valid) {
        if (idx < kStatParts) ws.pidx[idx] = ep[h];
#pragma unroll
        for (int g = 0; g < kTcMaxG; ++g) {
          if (g < G) {
            const float mk = em[h][g], lk = el[h][g];
            if (idx < kStatParts) ws.pm[idx][g] = mk;
            if (mk > -INFINITY) {
              const float mn = fmaxf(m[g], mk);
              l[g] = l[g] * ex2_approx(m[g] - mn) + lk * ex2_approx(mk - mn);
              m[g] = mn;
            }
          }
        }
      }
    }
  }
  float M[kTcMaxG], L[kTcMaxG];
#pragma unroll
  for (int g = 0; g < kTcMaxG; ++g) M[g] = m[g];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)  // all heads at once: independent shuffle chains
#pragma unroll
    for (int g = 0; g < kTcMaxG; ++g) M[g] = fmaxf(M[g], __shfl_xor_sync(0xffffffffu, M[g], off));
#pragma unroll
  for (int g = 0; g < kTcMaxG; ++g) L[g] = m[g] > -INFINITY ? l[g] * ex2_approx(m[g] - M[g]) : 0.f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
#pragma unroll
    for (int g = 0; g < kTcMaxG; ++g) L[g] += __shfl_xor_sync(0xffffffffu, L[g], off);
  if (lane < G) {  // lane g publishes head g
    float Mg = M[0], Lg = L[0];
#pragma unroll
    for (int g = 1; g < kTcMaxG; ++g)
      if (lane == g) {
        Mg = M[g];
        Lg = L[g];
      }
    ws.M[lane] = Mg;
    ws.Li[lane] = Lg > 0.f ? 1.f / Lg : 0.f;
    ws.lse[lane] = Mg + log2f(Lg);
  }
  if (lane == 0) ws.nr = found;
  __syncwarp();
}

// Step constants of `row` except its log-denominators (they need the step's
// partials): slot range, count, next free slot, the appended position, the
// recent-window threshold, budget checks. Run by one thread.
__device__ __forceinline__ void row_consts(const DecArgs& a, int row, RowC& R) {
  const int32_t* meta = a.meta + (long long)row * 8;
  const int count = meta[0], next = meta[1], steps = meta[2], count0 = meta[4];
  const long long base = a.slot_off[row];
  const int cap = (int)(a.slot_off[row + 1] - base);
  const int bb = a.b[row];
  const int n = count + 1;
  const int Mr = (a.recent_pct * bb) / 100;
  const int appended = steps + 1;
  const bool evict = n > bb;
  const bool ok = count < cap && next >= 0 && next < cap && (!evict || bb >= a.T + Mr);
  const int pos_new = row_len(a.map, row) + steps;
  // the M most recent positions are >= pos_thr: the appended ones and, early on,
  // the last prefill entries (never evicted while recent, so their pos is stable)
  int pos_thr = pos_new - Mr + 1;
  if (ok && appended < Mr && kv_check(count0 - (Mr - appended) < cap))
    pos_thr = a.pos[base + max(0, count0 - (Mr - appended))];
  R.base = base;
  R.cap = cap;
  R.n = n;
  R.next = next;
  R.pos_new = pos_new;
  R.pos_thr = pos_thr;
  R.bb = bb;
  R.steps = steps;
  R.target = (unsigned)(steps + 1) * (unsigned)cap;
  R.flags = (ok ? 1 : 0) | (evict ? 2 : 0);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) decode_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                const __grid_constant__ CUtensorMap tmV,
                                                                const __grid_constant__ CUtensorMap tmQ,
                                                                const __grid_constant__ TcArgs P) {
  constexpr int NDC = D / 16;             // 16-wide chunks of d
  constexpr int TILE = kTcSlots * D * 2;  // bytes of one K or V tile
  constexpr int STAGE = 2 * TILE + kQBytes;
  static_assert(kRowsBatch * (sizeof(RowStat) + sizeof(RowC)) <= kStages * STAGE, "finish scratch");
  const DecArgs& a = P.a;
  const TcScratch& sc = P.sc;
  const int G = a.G;
  const int n_rows = a.map.n_rows;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = warp >> 2, gt = tid & 127;

  extern __shared__ uint8_t dsm_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  float* o_s = reinterpret_cast<float*>(ring + kStages * STAGE);  // [groups][G][D]
  __shared__ uint64_t full[kStages];
  __shared__ TileHdr hdr[kStages];
  __shared__ float red_m[kWarps][kTcMaxG], red_l[kWarps][kTcMaxG];
  __shared__ int abort_s;
  __shared__ RowC rowc[kRowsBatch];   // constants of the first rows of this CTA's finish range
  __shared__ long long rng_s[2];      // the finish range [S0, S1) of slots
  __shared__ int rlo_s, rhi_s;        // its first and last row
  __shared__ int own_s;               // first row whose attention output this CTA writes
  // a group's current segment: slots attended, the row's step, the segment's first item in the row
  __shared__ int segc_s[kGroups], segs_s[kGroups], segk_s[kGroups];
  // a group's finished segments whose slot counts are published together at the end
  constexpr int kDefer = 16;
  __shared__ int dq_row[kGroups][kDefer], dq_cnt[kGroups][kDefer], dq_n[kGroups];
  __shared__ Walk walk_s[kGroups];  // each group's tile walk (its first thread's), kept out of registers
  __shared__ int more_s[kGroups], ended_s[kGroups], nreal_s[kGroups];
  __shared__ unsigned long long owns_s[kGroups];  // each group's unclaimed items (front, back)

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&full[i], 1);
    abort_s = 0;
    for (int g = 0; g < kGroups; ++g) dq_n[g] = 0;
    fence_barrier_init();
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmQ);
  }
  for (int i = tid; i < kGroups * G * D; i += kThreads) o_s[i] = 0.f;
  pdl_wait();  // the previous step has finished with the cache and the scratch
  pdl_launch_dependents();
  __syncthreads();
  const Guard gd{&abort_s, a.status, P.limit_ns};
  const int maxp = sc.max_per_row * kGroups;
  const int n_items = *sc.n_items;
  // this CTA's run of items: cut by cost at decode init for this grid, else equal counts
  int u0, u1;
  if (sc.cta_u[kMaxCtas] == (int)gridDim.x) {
    u0 = sc.cta_u[blockIdx.x];
    u1 = sc.cta_u[blockIdx.x + 1];
  } else {
    u0 = (int)((long long)n_items * blockIdx.x / gridDim.x);
    u1 = (int)((long long)n_items * (blockIdx.x + 1) / gridDim.x);
  }
  if (tid == 0)  // each group starts with a contiguous third of the CTA's items
    for (int g = 0; g < kGroups; ++g)
      owns_s[g] = pack_range(u0 + (int)((long long)(u1 - u0) * g / kGroups),
                             u0 + (int)((long long)(u1 - u0) * (g + 1) / kGroups));
  __syncthreads();

  // ---------------------------------------------------------------- attention
  {
    Walk& w = walk_s[grp];
    if (gt == 0) {
      const uint64_t stream_policy = make_policy_evict_first();  // K and V are read once per step
      int more = group_take(w, a, sc, owns_s, grp);
      int ended = 0, n_real = 0;
      for (int s = 0; s < kGStages && !ended; ++s) {
        const int stg = grp * kGStages + s;
        if (more) {
          issue_tile<D>(w, ring + stg * STAGE, &full[stg], &hdr[stg], &tmK, &tmV, &tmQ, a, stream_policy);
          ++n_real;
          more = walk_advance(w, a, sc.max_per_row, owns_s + grp) || group_take(w, a, sc, owns_s, grp);
        } else {
          hdr[stg].row = -1;
          mbar_arrive(&full[stg]);
          ended = 1;
        }
      }
      more_s[grp] = more;
      ended_s[grp] = ended;
      nreal_s[grp] = n_real;
    }
    if (warp == 0 && u0 < u1) {
      // this CTA's finish range and its rows' step constants, loaded while the
      // first tiles are in flight
      if (lane == 0) {
        const int2 i0 = sc.items[u0], i1 = sc.items[u1 - 1];
        const long long hb = a.slot_off[i1.x];
        rng_s[0] = a.slot_off[i0.x] + (long long)i0.y * kCH;
        rng_s[1] = hb + min((long long)(i1.y + 1) * kCH, a.slot_off[i1.x + 1] - hb);
        rlo_s = i0.x;
        rhi_s = i1.x;
        own_s = i0.y == 0 ? i0.x : i0.x + 1;  // rows whose first item is in this range
      }
      __syncwarp();
      const int rn = min(kRowsBatch, rhi_s - rlo_s + 1);
      for (int i = lane; i < rn; i += 32) row_consts(a, rlo_s + i, rowc[i]);
    }

    const int g0 = lane >> 2, q4 = lane & 3;  // this lane's query row and column pair
    const bool g_ok = g0 < G;
    const int m_ = lane >> 3, r_ = lane & 7;
    const int wslot = (warp & 3) * 16;  // this warp's 16 slots of a tile
    const uint64_t keep_policy = make_policy_evict_last();  // logits are read back after the barrier
    float* og = o_s + grp * G * D;
    bool aborted = false;
    int cur_row = -1, seg_u = -1;
    float m0 = -INFINITY, l0 = 0.f;
    float o[2 * NDC][2];  // O[g0][8 i + 2 q4 + {0,1}]
#pragma unroll
    for (int i = 0; i < 2 * NDC; ++i) o[i][0] = o[i][1] = 0.f;

    int k = 0;
    for (;; ++k) {
      const int stg = grp * kGStages + (k & 1);
      // the group decides together whether the stage arrived (its warps' barriers
      // and warp-wide instructions must not part)
      const bool got = named_bar_and(1 + grp, 128, !aborted && wait_bounded(&full[stg], (k >> 1) & 1, gd));
      if (!got) aborted = true;
      const int hrow = got ? hdr[stg].row : -1;  // -1: sentinel (or abort)
      if (hrow != cur_row || hrow < 0) {
        if (cur_row >= 0) {
          // leaving a row: the group's running (max, sum, O) becomes one partial at
          // (first item of the segment, group), listed for the row
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
          const int pidx = seg_u * kGroups + grp;
          float* part = sc.part + (long long)pidx * sc.stride;
          // the row's list place of this partial: (the segment's first item in the row, group)
          const int kk = segk_s[grp] * kGroups + grp;
          PEnt* ent = reinterpret_cast<PEnt*>(sc.plist) + (long long)cur_row * maxp + kk;
          if (gt < G) {
            float M = -INFINITY;
            for (int w4 = 0; w4 < 4; ++w4) M = fmaxf(M, red_m[grp * 4 + w4][gt]);
            float Ls = 0.f;
            for (int w4 = 0; w4 < 4; ++w4)
              if (red_m[grp * 4 + w4][gt] > -INFINITY)
                Ls += red_l[grp * 4 + w4][gt] * ex2_approx(red_m[grp * 4 + w4][gt] - M);
            part[gt] = M;
            part[G + gt] = Ls;
            if (kk < maxp) {
              ent->m[gt] = M;
              ent->l[gt] = Ls;
            }
          }
          if (gt == 0 && kk < maxp) {
            ent->pidx = pidx;
            ent->stamp = segs_s[grp] + 1;
          }
          // the group's warps add their O in four turns; in turn t warp w adds its quarter
          // (w + t) mod 4 of the columns, so every turn all four warps work and each
          // column still receives the warps in a fixed order (the step's result does not
          // depend on scheduling); in the last turn a column's sum is complete and goes
          // to the partial, and the buffer is cleared; lanes own distinct columns
          constexpr int QI = 2 * NDC / 4;  // i-values of a quarter
          for (int t4 = 0; t4 < 4; ++t4) {
            if (g_ok) {
              const int qb = ((warp & 3) + t4) & 3;
              float* ogp = og + g0 * D;
              float* pgp = part + kPartO + g0 * D;
              asm volatile("" : "+l"(ogp), "+l"(pgp));  // addresses formed here, not held across the turns
#pragma unroll
              for (int b = 0; b < 4; ++b)
                if (b == qb) {
#pragma unroll
                  for (int ii = 0; ii < QI; ++ii) {
                    const int i = b * QI + ii;
                    const int col = i * 8 + q4 * 2;
                    const int c0 = ogswz(g0, col), c1 = ogswz(g0, col + 1);
                    if (t4 < 3) {
                      ogp[c0] += o[i][0] * f0;
                      ogp[c1] += o[i][1] * f0;
                    } else {
                      *reinterpret_cast<float2*>(pgp + col) = make_float2(ogp[c0] + o[i][0] * f0, ogp[c1] + o[i][1] * f0);
                      ogp[c0] = 0.f;
                      ogp[c1] = 0.f;
                    }
                  }
                }
            }
            named_bar_sync(1 + grp, 128);  // after the last turn: the partial is written
          }
          if (gt == 0) {  // count the slots the partial covers, once it is visible (at the end)
            const int qn = dq_n[grp];
            if (qn < kDefer) {
              dq_row[grp][qn] = cur_row;
              dq_cnt[grp][qn] = segc_s[grp];
              dq_n[grp] = qn + 1;
            } else {
              __threadfence();
              atomicAdd(&sc.attn_done[cur_row], (unsigned)segc_s[grp]);
            }
          }
          m0 = -INFINITY;
          l0 = 0.f;
#pragma unroll
          for (int i = 0; i < 2 * NDC; ++i) o[i][0] = o[i][1] = 0.f;
        }
        if (hrow < 0) break;
        cur_row = hrow;
        seg_u = hdr[stg].u;
        if (gt == 0) {
          segs_s[grp] = hdr[stg].steps;
          segc_s[grp] = 0;
          segk_s[grp] = hdr[stg].st0 / kCH;
        }
      }
      const TileHdr h = hdr[stg];
      if (gt == 0) segc_s[grp] += min(h.st0 + kTcSlots, h.c1) - h.st0;
      uint8_t* stage = ring + stg * STAGE;
      const uint32_t ktile = smem_u32(stage), vtile = ktile + TILE;
      const int n = h.count + 1;
      const bool row_ok = h.count >= 0 && h.count < h.cap && h.next >= 0 && h.next < h.cap;
      const long long base = h.base;
      if (row_ok && h.next >= h.st0 + wslot && h.next < h.st0 + wslot + 16 && h.next < h.c1) {
        // the appended token: patch its K and V rows into the tile, write them to the cache
        const int r = h.next - h.st0;
        const __nv_bfloat16* kin = static_cast<const __nv_bfloat16*>(a.k) + (long long)h.row * D;
        const __nv_bfloat16* vin = static_cast<const __nv_bfloat16*>(a.v) + (long long)h.row * D;
        if (lane < D / 8) {
          const uint4 kv = *reinterpret_cast<const uint4*>(kin + lane * 8);
          const uint4 vv = *reinterpret_cast<const uint4*>(vin + lane * 8);
          *reinterpret_cast<uint4*>(stage + (swz(ktile, r, lane * 8) - ktile)) = kv;
          *reinterpret_cast<uint4*>(stage + (swz(vtile, r, lane * 8) - ktile)) = vv;
          reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.Kc) + (base + h.next) * D)[lane] = kv;
          reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.Vc) + (base + h.next) * D)[lane] = vv;
        }
        if (lane == 0) a.pos[base + h.next] = row_len(a.map, h.row) + h.steps;
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
        uint32_t b00, b01, b10, b11, q0, q1;
        ldsm_x2(qswz(qarea, qrow, dc * 16 + ((lane >> 3) & 1) * 8), q0, q1);
        ldsm_x4(swz(ktile, wslot + (m_ >> 1) * 8 + r_, dc * 16 + (m_ & 1) * 8), b00, b01, b10, b11);
        const uint32_t af[4] = {g_ok ? q0 : 0u, 0u, g_ok ? q1 : 0u, 0u};
        if (dc & 1) {
          mma16816(t0, af, b00, b01);
          mma16816(t1, af, b10, b11);
        } else {
          mma16816(s0, af, b00, b01);
          mma16816(s1, af, b10, b11);
        }
      }
      const int jb = h.st0 + wslot + q4 * 2;  // slots jb, jb+1 (n-tile 0) and jb+8, jb+9 (n-tile 1)
      float x[4];                              // row g0 at those four slots
      x[0] = s0[0] + t0[0];
      x[1] = s0[1] + t0[1];
      x[2] = s1[0] + t1[0];
      x[3] = s1[1] + t1[1];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = jb + (e & 1) + (e >> 1) * 8;
        const bool valid = row_ok && j < n && j < h.c1;
        x[e] = valid ? x[e] * a.scale2 : -INFINITY;
        // eight logits per slot: the lanes of heads >= G store -inf, so the finish
        // reads every slot's logits as two aligned float4 whatever G is
        if (valid) st_f32_hint(sc.logits + (base + j) * kTcMaxG + g0, g_ok ? x[e] : -INFINITY, keep_policy);
      }
      // online softmax update of this warp's running (max, sum, O)
      float tm = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
      tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 1));
      tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 2));
      const float nm = fmaxf(m0, tm);
      const float vm = nm == -INFINITY ? 0.f : nm;
      if (__any_sync(0xffffffffu, nm != m0)) {  // rescale only when a running max moved
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
      if (gt == 0) {
        if (more_s[grp]) {
          issue_tile<D>(w, stage, &full[stg], &hdr[stg], &tmK, &tmV, &tmQ, a, make_policy_evict_first());
          ++nreal_s[grp];
          more_s[grp] = walk_advance(w, a, sc.max_per_row, owns_s + grp) || group_take(w, a, sc, owns_s, grp);
        } else if (!ended_s[grp]) {
          hdr[stg].row = -1;
          mbar_arrive(&full[stg]);
          ended_s[grp] = 1;
        }
      }
    }
    if (gt == 0 && dq_n[grp] > 0) {  // publish the group's partials, then their slot counts
      __threadfence();
      for (int i = 0; i < dq_n[grp]; ++i) atomicAdd(&sc.attn_done[dq_row[grp][i]], (unsigned)dq_cnt[grp][i]);
    }
    if (aborted) {
      abort_s = 1;
      if (gt == 0)  // let this group's copies in flight land before the CTA exits
        for (int t = k; t < nreal_s[grp]; ++t) wait_drain(&full[grp * kGStages + (t & 1)], (t >> 1) & 1);
    }
  }
  __syncthreads();

  // ------------------------------------------------------------------ finish
  // A row is finished by the CTAs whose ranges hold its slots, once every CTA
  // has attended its part of the row (the row's attended-slot count reaches
  // its target; the wait is bounded). No CTA waits for rows outside its range.
  __syncthreads();
  if (u0 >= u1 || abort_s) return;
  RowStat* rs = reinterpret_cast<RowStat*>(ring);  // the tile ring is free now
  RowC* rcb = reinterpret_cast<RowC*>(ring + kRowsBatch * sizeof(RowStat));
  const int E = G * D;
  const int nq = (E + kOutUnit - 1) / kOutUnit;
  const int r_lo = rlo_s, r_hi = rhi_s, own_lo = own_s;
  const long long S0 = rng_s[0], S1 = rng_s[1];
  constexpr int UP = 6;  // slots per lane in flight in the sweep
  // The first batch's slot data (logits written by this CTA, A, positions: none of it
  // waits for another CTA) is copied into the rest of the freed ring now, without
  // waiting; the sweep reads it from there.
  constexpr size_t kStgOff = (size_t)kRowsBatch * (sizeof(RowStat) + sizeof(RowC));
  constexpr int kStgSlots = (int)(((size_t)kStages * STAGE - kStgOff) / 40);
  static_assert(kStgOff % 16 == 0, "staging alignment");
  float* st_lg = reinterpret_cast<float*>(ring + kStgOff);  // [kStgSlots][8]
  float* st_A = st_lg + (size_t)kStgSlots * kTcMaxG;        // [kStgSlots]
  int* st_pos = reinterpret_cast<int*>(st_A + kStgSlots);    // [kStgSlots]
  long long stg0 = 0;
  int nst = 0;
  {
    const int rn0 = min(kRowsBatch, r_hi - r_lo + 1);
    stg0 = max(S0, rowc[0].base);
    const long long stg1 = min(S1, rowc[rn0 - 1].base + rowc[rn0 - 1].cap);
    nst = (int)max(0ll, min(stg1 - stg0, (long long)kStgSlots));
    const float* lsrc = sc.logits + stg0 * kTcMaxG;
    for (int i = tid; i < nst * 2; i += kThreads) cp_async16(st_lg + i * 4, lsrc + i * 4);
    for (int i = tid; i < nst; i += kThreads) {
      cp_async4(st_A + i, a.A + stg0 + i);
      cp_async4(st_pos + i, a.pos + stg0 + i);
    }
  }
  for (int rb = r_lo; rb <= r_hi; rb += kRowsBatch) {
    const int rn = min(kRowsBatch, r_hi - rb + 1);
    RowC* rc = rb == r_lo ? rowc : rcb;
    // (1) per row (one warp each): wait for the row's attention, then its log-denominators
    for (int i = warp; i < rn; i += kWarps) {
      const int row = rb + i;
      if (rb != r_lo && lane == 0) row_consts(a, row, rc[i]);
      __syncwarp();
      int waited = 1;
      if (lane == 0) {
        const volatile unsigned* cnt = sc.attn_done + row;
        const unsigned target = rc[i].target;
        if ((int)(*cnt - target) < 0) {
          const uint64_t t0 = globaltimer();
          while ((int)(*cnt - target) < 0) {
            if (globaltimer() - t0 > P.limit_ns) {
              atomicOr(a.status, KV_DEV_TIMEOUT);
              waited = 0;
              break;
            }
          }
        }
        __threadfence();
      }
      waited = __shfl_sync(0xffffffffu, waited, 0);
      if (!waited) abort_s = 1;
      row_stats(P, row, ((rc[i].cap + kCH - 1) / kCH) * kGroups, rc[i].steps + 1, lane, rs[i]);
    }
    cp_async_wait_all();  // this thread's copies into the staging area
    __syncthreads();      // ... and everyone else's
    if (abort_s) return;

    // (2) decayed scores and evictions first: this warp's share of the batch's slots within the range
    const long long B0 = max(S0, rc[0].base), B1 = min(S1, rc[rn - 1].base + rc[rn - 1].cap);
    const long long len = B1 > B0 ? B1 - B0 : 0;
    const long long w0 = B0 + len * warp / kWarps, w1 = B0 + len * (warp + 1) / kWarps;
    int ri = 0;
    while (ri < rn - 1 && w0 >= rc[ri].base + rc[ri].cap) ++ri;
    for (long long p0 = w0; p0 < w1; ++ri) {
      const RowC& R = rc[ri];
      const long long p1 = min(w1, R.base + R.cap);
      const int row = rb + ri;
      const bool ok = (R.flags & 1) != 0;
      Best best{INFINITY, -1, -1};
      if (ok) {
        const uint64_t keep = make_policy_evict_last();
        const long long rbase = R.base;  // register copies for the sweep
        const int rn_ = R.n, rnext = R.next, rpos_new = R.pos_new, rpos_thr = R.pos_thr;
        float lse[kTcMaxG];
#pragma unroll
        for (int g = 0; g < kTcMaxG; ++g) lse[g] = g < G ? rs[ri].lse[g] : 0.f;
        // one slot per lane (all eight logits, A and the position), U slots per lane
        // with every load issued before the first use
        constexpr int U = UP;
        for (long long s0 = p0; s0 < p1; s0 += 32 * U) {
          float4 la[U], lb[U];
          float Av[U];
          int pv[U];
          if (s0 >= stg0 && min(s0 + 32 * U, p1) <= stg0 + nst) {  // staged in shared memory
#pragma unroll
            for (int uu = 0; uu < U; ++uu) {
              const int k = (int)(min(s0 + uu * 32 + lane, p1 - 1) - stg0);
              la[uu] = *reinterpret_cast<const float4*>(st_lg + k * kTcMaxG);
              lb[uu] = *reinterpret_cast<const float4*>(st_lg + k * kTcMaxG + 4);
              Av[uu] = st_A[k];
              pv[uu] = st_pos[k];
            }
          } else {
#pragma unroll
            for (int uu = 0; uu < U; ++uu) {  // every load first, addresses clamped into the piece
              const long long s = min(s0 + uu * 32 + lane, p1 - 1);
              la[uu] = __ldcg(reinterpret_cast<const float4*>(sc.logits + s * kTcMaxG));
              lb[uu] = __ldcg(reinterpret_cast<const float4*>(sc.logits + s * kTcMaxG) + 1);
              Av[uu] = __ldcg(a.A + s);
              pv[uu] = __ldcg(a.pos + s);
            }
          }
          const int jb = (int)(s0 - rbase) + lane;
#pragma unroll
          for (int uu = 0; uu < U; ++uu) {
            const float ps =
                (((ex2_approx(la[uu].x - lse[0]) + ex2_approx(la[uu].y - lse[1])) + ex2_approx(la[uu].z - lse[2])) +
                 ex2_approx(la[uu].w - lse[3])) +
                (((ex2_approx(lb[uu].x - lse[4]) + ex2_approx(lb[uu].y - lse[5])) + ex2_approx(lb[uu].z - lse[6])) +
                 ex2_approx(lb[uu].w - lse[7]));
            const int j = jb + uu * 32;
            if (j < (int)(p1 - rbase) && j < rn_) {
              const float Anew = (j == rnext ? 0.f : a.gamma * Av[uu]) + ps;
              st_f32_hint_nc(a.A + rbase + j, Anew, keep);  // read again by the next step
              const int pj = j == rnext ? rpos_new : pv[uu];
              if (j >= a.T && pj < rpos_thr) {
                const Best c{Anew, pj, j};
                if (better(c, best)) best = c;
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
      int last = 0;
      if (lane == 0) {
        if (best.slot >= 0) {
          const int idx = atomicAdd(&sc.best_n[row], 1);
          if (idx < sc.max_bests)
            sc.bests[(long long)row * sc.max_bests + idx] = make_int4(__float_as_int(best.A), best.pos, best.slot, 0);
        }
        __threadfence();
        const int cnt = (int)(p1 - p0);
        last = atomicAdd(&sc.done[row], cnt) + cnt == R.cap;
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {  // every slot of the row is done: pick the eviction, write the row's meta data
        __threadfence();
        const int nb = __ldcg(sc.best_n + row);
        Best bst{INFINITY, -1, -1};
        for (int kb = lane; kb < min(nb, sc.max_bests); kb += 32) {
          const int4 v = __ldcg(sc.bests + (long long)row * sc.max_bests + kb);
          const Best c{__int_as_float(v.x), v.y, v.z};
          if (better(c, bst)) bst = c;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          Best y;
          y.A = __shfl_xor_sync(0xffffffffu, bst.A, off);
          y.pos = __shfl_xor_sync(0xffffffffu, bst.pos, off);
          y.slot = __shfl_xor_sync(0xffffffffu, bst.slot, off);
          if (better(y, bst)) bst = y;
        }
        if (lane == 0) {
          int32_t* meta = a.meta + (long long)row * 8;
          if (!ok) {
            atomicOr(a.status, KV_DEV_BUDGET);
          } else if ((R.flags & 4) || nb > sc.max_bests) {
            atomicOr(a.status, KV_DEV_CAPACITY);
          } else {
            if ((R.flags & 2) && bst.slot >= 0 && kv_check(bst.slot < R.cap)) {
              meta[0] = R.bb;
              meta[1] = bst.slot;
              meta[3] = bst.slot;
            } else {
              meta[0] = R.n;
              meta[1] = R.n;
              meta[3] = -1;
            }
            meta[2] = R.steps + 1;
          }
          sc.done[row] = 0;
          sc.best_n[row] = 0;
        }
      }
      p0 = p1;
    }
    // (3) attention outputs of the rows whose first item is in this range: units of
    // kOutUnit elements over the warps, from the last warp down (after the sweep: the
    // next step waits for the evictions, not for the outputs)
    const int o_first = max(rb, own_lo) - rb;
    const int n_units = max(0, rn - o_first) * nq;
    for (int un = kWarps - 1 - warp; un < n_units; un += kWarps) {
      const int i = o_first + un / nq, q = un % nq;
      const int row = rb + i;
      const RowStat& st = rs[i];
      const int nr = st.nr;
      // lane: elements e0..e0+3 and e0+128..e0+131 of the unit, so each of the warp's
      // two loads per partial is 512 contiguous bytes
      const int e0 = q * kOutUnit + lane * 4, e1 = e0 + kOutUnit / 2;
      const bool ok0 = e0 < E, ok1 = e1 < E;
      const int g0 = ok0 ? e0 / D : 0, g1 = ok1 ? e1 / D : 0;
      const float M0 = st.M[g0], M1 = st.M[g1];
      const PEnt* lst = reinterpret_cast<const PEnt*>(sc.plist) + (long long)row * maxp;
      const int stamp = rc[i].steps + 1, ncand = min(((rc[i].cap + kCH - 1) / kCH) * kGroups, maxp);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      auto add = [&](int pi, float mk0, float mk1) {
        const float* pc = sc.part + (long long)pi * sc.stride + kPartO;
        const float4 v0 = ok0 ? __ldcg(reinterpret_cast<const float4*>(pc + e0)) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 v1 = ok1 ? __ldcg(reinterpret_cast<const float4*>(pc + e1)) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float w0 = mk0 > -INFINITY ? ex2_approx(mk0 - M0) : 0.f;
        const float w1 = mk1 > -INFINITY ? ex2_approx(mk1 - M1) : 0.f;
        acc[0] += w0 * v0.x;
        acc[1] += w0 * v0.y;
        acc[2] += w0 * v0.z;
        acc[3] += w0 * v0.w;
        acc[4] += w1 * v1.x;
        acc[5] += w1 * v1.y;
        acc[6] += w1 * v1.z;
        acc[7] += w1 * v1.w;
      };
      if (nr <= kStatParts) {
#pragma unroll 8
        for (int kp = 0; kp < nr; ++kp) add(st.pidx[kp], st.pm[kp][g0], st.pm[kp][g1]);
      } else {  // more partials than held on chip: read every place again
        for (int kp = 0; kp < ncand; ++kp)
          if (__ldcg(&lst[kp].stamp) == stamp) add(__ldcg(&lst[kp].pidx), __ldcg(&lst[kp].m[g0]), __ldcg(&lst[kp].m[g1]));
      }
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) + (long long)row * E;
      if (ok0) {
        const float li = st.Li[g0];
        uint2 pk;
        pk.x = pack_bf16(acc[0] * li, acc[1] * li);
        pk.y = pack_bf16(acc[2] * li, acc[3] * li);
        *reinterpret_cast<uint2*>(orow + e0) = pk;
      }
      if (ok1) {
        const float li = st.Li[g1];
        uint2 pk;
        pk.x = pack_bf16(acc[4] * li, acc[5] * li);
        pk.y = pack_bf16(acc[6] * li, acc[7] * li);
        *reinterpret_cast<uint2*>(orow + e1) = pk;
      }
    }

    __syncthreads();  // the row statistics and constants are rewritten by the next batch
  }
}

}  // namespace

size_t tc_scratch_bytes(const kv_shape& sh, const RowMap& m, int capb, long long total_slots) {
  return tc_layout(m.n_rows, sh.group, sh.head_dim, capb, total_slots, nullptr, nullptr);
}

int launch_tc_init(const kv_shape& sh, const RowMap& m, int capb, long long total_slots, const kv_cache& c,
                   cudaStream_t st) {
  TcScratch sc;
  const size_t need = tc_layout(m.n_rows, sh.group, sh.head_dim, capb, total_slots, (char*)c.scratch, &sc);
  if (!c.scratch || c.scratch_bytes < need) return KV_ERR_WORKSPACE;
  // list entries carry the step they belong to: clear the stamps of any earlier decode
  if (cudaMemsetAsync(sc.plist, 0, (size_t)m.n_rows * sc.max_per_row * kGroups * sizeof(PEnt), st) != cudaSuccess)
    return KV_ERR_CUDA;
  const int n_cta = std::min(sm_count(), kMaxCtas);  // the decode grid (one CTA per SM)
  tc_items_kernel<<<1, 1024, 0, st>>>(m.n_rows, c.slot_off, sc, n_cta, c.status);
  return cuda_status(cudaGetLastError());
}

int launch_tc(const kv_shape& sh, const RowMap& m, int capb, long long total_slots, const DecArgs& a,
              const kv_cache& c, cudaStream_t st) {
  if (total_slots >= (1ll << 31)) return KV_ERR_ARG;  // slot indices are TMA coordinates (int32)
  TcArgs P;
  P.a = a;
  P.limit_ns = wait_limit_ns();
  const size_t need = tc_layout(m.n_rows, sh.group, sh.head_dim, capb, total_slots, (char*)c.scratch, &P.sc);
  if (!c.scratch || c.scratch_bytes < need) return KV_ERR_WORKSPACE;
  const int stage_bytes = 2 * kTcSlots * sh.head_dim * 2 + kQBytes;
  const size_t smem = 1024 + (size_t)kStages * stage_bytes + (size_t)kGroups * sh.group * sh.head_dim * 4;
  CUtensorMap tmK, tmV, tmQ;
  if (!encode_rows_bf16(&tmK, c.Kc, sh.head_dim, total_slots, kTcSlots)) return KV_ERR_CUDA;
  if (!encode_rows_bf16(&tmV, c.Vc, sh.head_dim, total_slots, kTcSlots)) return KV_ERR_CUDA;
  if (!encode_rows_bf16(&tmQ, a.q, sh.head_dim, (long long)m.n_rows * sh.group, sh.group)) return KV_ERR_CUDA;
  auto kern = sh.head_dim == 128 ? decode_tc_kernel<128> : decode_tc_kernel<64>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return KV_ERR_ARG;
  // the launch may start while the previous step's kernel drains (programmatic
  // dependent launch); it waits (griddepcontrol.wait) before touching memory
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(std::min(sm_count(), kMaxCtas));  // one CTA per SM (shared memory), all resident
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, tmK, tmV, tmQ, P));
}

}  // namespace kvc
