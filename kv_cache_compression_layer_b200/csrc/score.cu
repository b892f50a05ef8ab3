// kv_score: observation-window importance scores (AudioKV blog §1.2, the raw
// importance scores that Spectral Score Smoothing later smooths):
//   s_j = sum_{r<R} softmax_j(q_r . K_j / sqrt(d)),  R = g * w window rows.
//
// bf16 path (tcgen05 + TMEM + TMA), two passes over K with a tiny merge:
//   pass 1  D[r][j] = Q K_tile^T on the tensor core (M = 128 window rows per
//           half, N = 128 keys); the epilogue turns each row of the tile into
//           (tile max m, sum of exp2((x - m) c)) partials.
//   merge   per (row, r): lse2_r = log2 of the softmax denominator (c = log2 e
//           / sqrt d units), from the tile partials.
//   pass 2  D[j][r] = K_tile Q^T (M = 128 keys, N = R); each epilogue thread
//           owns one key and sums exp2(x c - lse2_r) over the R window rows.
// Both passes are persistent (one CTA per SM, contiguous runs of tiles) and
// warp-specialised: warp 0 issues TMA loads of Q and a 4-stage ring of K
// tiles, warp 1 issues tcgen05.mma into a double-buffered TMEM accumulator,
// warps 2-9 (two groups of four, one group per accumulator buffer) read TMEM
// with tcgen05.ld and do the softmax arithmetic.
//
// fp32 path (fp32 inputs): the same three steps on CUDA cores (FFMA), since
// a tf32 contraction would not meet the fp32 tolerance.
#include <cmath>
#include <mutex>

#include "internal.h"

namespace kvc {
namespace {

constexpr int kStages = 4;
constexpr int kQRows = 256;
constexpr int kThreads = 320;
constexpr int kQChunkBytes = kQRows * 128;      // 256 rows x 64 bf16
constexpr int kKChunkBytes = kTileKeys * 128;   // 128 keys x 64 bf16
constexpr int kKStageBytes = 2 * kKChunkBytes;  // d <= 128
constexpr int kSmemQ = 0;
constexpr int kSmemK = 2 * kQChunkBytes;
constexpr int kSmemBar = kSmemK + kStages * kKStageBytes;
constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 1;
constexpr int kSmemMisc = kSmemBar + kNumBars * 8;
constexpr int kSmemTotal = kSmemMisc + 16;
constexpr int kSmemAlloc = kSmemTotal + 1024;  // slack for 1024-byte alignment

struct TcArgs {
  RowMap map;
  int R;      // valid window rows
  int n2;     // pass-2 MMA N: R rounded up to 16
  int nk;     // 64-element chunks of d (1 or 2)
  int total_tiles;
  float c;    // log2(e) / sqrt(d)
  float2* partial;     // pass 1 out: [total_tiles][R] (tile max, tile sum)
  const float* lse2;   // pass 2 in:  [rows][R]
  float* s;            // pass 2 out: [sum L]
  int* status;
  unsigned long long limit_ns;
};

template <int PASS>
__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kSmemQ;
  uint8_t* sK = smem + kSmemK;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBar);
  uint64_t* full_k = bars;
  uint64_t* empty_k = bars + kStages;
  uint64_t* q_full = bars + 2 * kStages;
  uint64_t* q_empty = q_full + 1;
  uint64_t* acc_full = q_full + 2;
  uint64_t* acc_empty = q_full + 4;
  uint64_t* drain = q_full + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSmemMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSmemMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int u0 = (int)((long long)a.total_tiles * blockIdx.x / G);
  const int u1 = (int)((long long)a.total_tiles * (blockIdx.x + 1) / G);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full_k[i], 1);
      mbar_init(&empty_k[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 1 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Guard g{abort_flag, a.status, a.limit_ns};

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0, cur_row = -1;
      uint32_t qe_phase = 0;
      bool have_q = false;
      bool k_issued[kStages] = {false, false, false, false};
      uint32_t k_parity[kStages] = {0, 0, 0, 0};
      uint32_t q_parity = 0;
      bool aborted = false;
      for (int u = u0; u < u1; ++u, ++it) {
        int row, tile;
        tile_to_row(a.map, u, row, tile);
        if (row != cur_row) {
          if (have_q) {
            if (!wait_bounded(q_empty, qe_phase, g)) { aborted = true; break; }
            qe_phase ^= 1;
            q_parity ^= 1;
          }
          have_q = true;
          cur_row = row;
          mbar_arrive_expect_tx(q_full, a.nk * kQChunkBytes);
          for (int c = 0; c < a.nk; ++c) tma_load_2d(sQ + c * kQChunkBytes, &tmQ, q_full, c * 64, row * a.R);
        }
        const int st = it % kStages;
        if (it >= kStages && !wait_bounded(&empty_k[st], ((it / kStages) - 1) & 1, g)) { aborted = true; break; }
        mbar_arrive_expect_tx(&full_k[st], a.nk * kKChunkBytes);
        const long long key0 = row_key_off(a.map, row) + (long long)tile * kTileKeys;
        for (int c = 0; c < a.nk; ++c)
          tma_load_2d(sK + st * kKStageBytes + c * kKChunkBytes, &tmK, &full_k[st], c * 64, (int)key0);
        k_issued[st] = true;
        k_parity[st] = (it / kStages) & 1;
      }
      if (aborted || *abort_flag) {
        // let the copies in flight land before the CTA's shared memory goes away
        for (int st = 0; st < kStages; ++st)
          if (k_issued[st]) wait_drain(&full_k[st], k_parity[st], a.limit_ns);
        if (have_q) wait_drain(q_full, q_parity, a.limit_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, cur_row = -1;
      uint32_t qf_phase = 0;
      const uint32_t qbase = smem_u32(sQ);
      for (int u = u0; u < u1; ++u, ++it) {
        int row, tile;
        tile_to_row(a.map, u, row, tile);
        if (row != cur_row) {
          if (!wait_bounded(q_full, qf_phase, g)) break;
          qf_phase ^= 1;
          cur_row = row;
        }
        const int st = it % kStages;
        if (!wait_bounded(&full_k[st], (it / kStages) & 1, g)) break;
        const int acc = it & 1;
        if (it >= 2 && !wait_bounded(&acc_empty[acc], ((it >> 1) - 1) & 1, g)) break;
        tc_fence_after();
        const uint32_t d_base = tmem + acc * 256;
        const uint32_t kbase = smem_u32(sK + st * kKStageBytes);
        if (PASS == 1) {
          const uint32_t idesc = idesc_bf16_f32(128, 128);
          for (int h = 0; h * 128 < a.R; ++h)
            for (int kk = 0; kk < a.nk * 4; ++kk) {
              const uint64_t ad = sw128_kmajor_desc(qbase + (kk >> 2) * kQChunkBytes + h * 128 * 128 + (kk & 3) * 32);
              const uint64_t bd = sw128_kmajor_desc(kbase + (kk >> 2) * kKChunkBytes + (kk & 3) * 32);
              tc_mma_bf16(d_base + h * 128, ad, bd, idesc, kk > 0);
            }
        } else {
          const uint32_t idesc = idesc_bf16_f32(128, a.n2);
          for (int kk = 0; kk < a.nk * 4; ++kk) {
            const uint64_t ad = sw128_kmajor_desc(kbase + (kk >> 2) * kKChunkBytes + (kk & 3) * 32);
            const uint64_t bd = sw128_kmajor_desc(qbase + (kk >> 2) * kQChunkBytes + (kk & 3) * 32);
            tc_mma_bf16(d_base, ad, bd, idesc, kk > 0);
          }
        }
        tc_commit(&empty_k[st]);
        tc_commit(&acc_full[acc]);
        int nrow = -1, ntile;
        if (u + 1 < u1) tile_to_row(a.map, u + 1, nrow, ntile);
        if (nrow != row) tc_commit(q_empty);
      }
      // every issued MMA has finished before TMEM is released
      tc_commit(drain);
      wait_drain(drain, 0, a.limit_ns);
    }
  } else {
    // ------------------------------------------------------ epilogue
    const int eg = (warp - 2) >> 2;  // accumulator buffer this group owns
    const int quarter = warp & 3;    // TMEM lanes [32 quarter, 32 quarter + 32)
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    for (int u = u0 + eg; u < u1; u += 2) {
      const int it = u - u0;
      int row, tile;
      tile_to_row(a.map, u, row, tile);
      const int nvalid = min(kTileKeys, row_len(a.map, row) - tile * kTileKeys);
      if (!wait_bounded(&acc_full[eg], (it >> 1) & 1, g)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + lane_addr + eg * 256;
      float x[4][32];
      if (PASS == 1) {
        for (int h = 0; h * 128 < a.R; ++h) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) tmem_ld32(tbase + h * 128 + cc * 32, x[cc]);
          tc_wait_ld();
          const bool last = (h + 1) * 128 >= a.R;
          if (last) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[eg]);
          }
          const int r = h * 128 + quarter * 32 + lane;
          float m = -INFINITY;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (cc * 32 + i < nvalid) m = fmaxf(m, x[cc][i]);
          const float mc = m * a.c;
          float Z = 0.f;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (cc * 32 + i < nvalid) Z += ex2_approx(fmaf(x[cc][i], a.c, -mc));
          if (r < a.R) a.partial[(long long)u * a.R + r] = make_float2(m, Z);
        }
      } else {
        const int j = quarter * 32 + lane;
        const float* lse = a.lse2 + (long long)row * a.R;
        float sum = 0.f;
        for (int cb = 0; cb * 128 < a.R; ++cb) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
            if (cb * 128 + cc * 32 < a.n2) tmem_ld32(tbase + cb * 128 + cc * 32, x[cc]);
          tc_wait_ld();
          if ((cb + 1) * 128 >= a.R) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[eg]);
          }
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const int col = cb * 128 + cc * 32;
            if (col < a.R) {
#pragma unroll
              for (int i = 0; i < 32; i += 4) {
                const float4 l4 = __ldg(reinterpret_cast<const float4*>(lse + col + i));
                sum += ex2_approx(fmaf(x[cc][i + 0], a.c, -l4.x));
                sum += ex2_approx(fmaf(x[cc][i + 1], a.c, -l4.y));
                sum += ex2_approx(fmaf(x[cc][i + 2], a.c, -l4.z));
                sum += ex2_approx(fmaf(x[cc][i + 3], a.c, -l4.w));
              }
            }
          }
        }
        if (j < nvalid) a.s[row_key_off(a.map, row) + (long long)tile * kTileKeys + j] = sum;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Softmax denominators of every (row, window row) from the tile partials.
__global__ void score_merge_kernel(const RowMap map, int R, float c, const float2* __restrict__ partial,
                                   float* __restrict__ lse2) {
  const int row = blockIdx.x, r = threadIdx.x;
  if (r >= R) return;
  const int s = row / map.rows_per_seq;
  const int tpr = (map.L[s] + kTileKeys - 1) / kTileKeys;
  const long long u_first = map.tile_off[s] + (long long)(row - s * map.rows_per_seq) * tpr;
  float m = -INFINITY, Z = 0.f;
  for (int t = 0; t < tpr; ++t) {
    const float2 p = partial[(u_first + t) * R + r];
    if (p.x > m) {
      Z = Z * exp2f((m - p.x) * c) + p.y;
      m = p.x;
    } else {
      Z += p.y * exp2f((p.x - m) * c);
    }
  }
  lse2[(long long)row * R + r] = m * c + log2f(Z);
}

// fp32 inputs: row statistics of one 128-key tile on CUDA cores.
__global__ void score_f32_stats_kernel(const RowMap map, int R, int d, float c, const float* __restrict__ qwin,
                                       const float* __restrict__ K, float2* __restrict__ partial) {
  extern __shared__ float fs[];
  const int dp = d + 1;
  float* Ks = fs;                  // [128][d+1]
  float* Qs = fs + kTileKeys * dp;  // [R][d+1]
  const int u = blockIdx.x;
  int row, tile;
  tile_to_row(map, u, row, tile);
  const int nvalid = min(kTileKeys, row_len(map, row) - tile * kTileKeys);
  const float* Kt = K + (row_key_off(map, row) + (long long)tile * kTileKeys) * d;
  for (int i = threadIdx.x; i < kTileKeys * d; i += blockDim.x) {
    const int j = i / d, k = i % d;
    Ks[j * dp + k] = j < nvalid ? Kt[(long long)j * d + k] : 0.f;
  }
  const float* Qr = qwin + (long long)row * R * d;
  for (int i = threadIdx.x; i < R * d; i += blockDim.x) Qs[(i / d) * dp + i % d] = Qr[i];
  __syncthreads();
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    float m = -INFINITY, Z = 0.f;
    for (int j = 0; j < nvalid; ++j) {
      float x = 0.f;
      for (int k = 0; k < d; ++k) x = fmaf(Qs[r * dp + k], Ks[j * dp + k], x);
      if (x > m) {
        Z = Z * ex2_approx((m - x) * c) + 1.f;
        m = x;
      } else {
        Z += ex2_approx((x - m) * c);
      }
    }
    partial[(long long)u * R + r] = make_float2(m, Z);
  }
}

// fp32 inputs: column sums of one 128-key tile on CUDA cores.
__global__ void score_f32_colsum_kernel(const RowMap map, int R, int d, float c, const float* __restrict__ qwin,
                                        const float* __restrict__ K, const float* __restrict__ lse2,
                                        float* __restrict__ s) {
  extern __shared__ float fs[];
  const int dp = d + 1;
  float* Ks = fs;
  float* Qs = fs + kTileKeys * dp;
  float* Ls = Qs + R * dp;
  const int u = blockIdx.x;
  int row, tile;
  tile_to_row(map, u, row, tile);
  const int nvalid = min(kTileKeys, row_len(map, row) - tile * kTileKeys);
  const long long key0 = row_key_off(map, row) + (long long)tile * kTileKeys;
  const float* Kt = K + key0 * d;
  for (int i = threadIdx.x; i < kTileKeys * d; i += blockDim.x) {
    const int j = i / d, k = i % d;
    Ks[j * dp + k] = j < nvalid ? Kt[(long long)j * d + k] : 0.f;
  }
  const float* Qr = qwin + (long long)row * R * d;
  for (int i = threadIdx.x; i < R * d; i += blockDim.x) Qs[(i / d) * dp + i % d] = Qr[i];
  for (int i = threadIdx.x; i < R; i += blockDim.x) Ls[i] = lse2[(long long)row * R + i];
  __syncthreads();
  const int j = threadIdx.x;
  if (j >= nvalid) return;
  float sum = 0.f;
  for (int r = 0; r < R; ++r) {
    float x = 0.f;
    for (int k = 0; k < d; ++k) x = fmaf(Qs[r * dp + k], Ks[j * dp + k], x);
    sum += ex2_approx(fmaf(x, c, -Ls[r]));
  }
  s[key0 + j] = sum;
}

}  // namespace

ScoreWs score_ws_layout(const RowMap& m, int R) {
  ScoreWs w;
  const long long tiles = m.tile_off[m.n_seq];
  w.status_off = 0;
  w.partial_off = 256;
  w.lse_off = w.partial_off + (((size_t)tiles * R * sizeof(float2) + 255) & ~size_t(255));
  w.bytes = w.lse_off + (((size_t)m.n_rows * R * sizeof(float) + 255) & ~size_t(255));
  return w;
}

int launch_score(const kv_shape& sh, const RowMap& m, const void* qwin, const void* K, float* s, void* ws,
                 cudaStream_t st) {
  const int R = sh.group * sh.w;
  const int d = sh.head_dim;
  const ScoreWs lay = score_ws_layout(m, R);
  char* wsb = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(wsb + lay.status_off);
  float2* partial = reinterpret_cast<float2*>(wsb + lay.partial_off);
  float* lse2 = reinterpret_cast<float*>(wsb + lay.lse_off);
  const int total_tiles = m.tile_off[m.n_seq];
  const float c = (float)(1.4426950408889634 / std::sqrt((double)d));
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return KV_ERR_CUDA;
  const int merge_threads = ((R + 31) / 32) * 32;

  if (sh.dtype == KV_BF16) {
    CUtensorMap tmQ, tmK;
    if (!encode_rows_bf16(&tmQ, qwin, d, (long long)m.n_rows * R, kQRows)) return KV_ERR_CUDA;
    if (!encode_rows_bf16(&tmK, K, d, total_keys(m), kTileKeys)) return KV_ERR_CUDA;
    static std::once_flag attr_once;
    std::call_once(attr_once, [] {
      cudaFuncSetAttribute(score_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
      cudaFuncSetAttribute(score_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    });
    TcArgs a;
    a.map = m;
    a.R = R;
    a.n2 = ((R + 15) / 16) * 16;
    a.nk = d / 64;
    a.total_tiles = total_tiles;
    a.c = c;
    a.partial = partial;
    a.lse2 = lse2;
    a.s = s;
    a.status = status;
    a.limit_ns = kWaitLimitNs;
    const int grid = std::min(sm_count(), total_tiles);
    score_tc_kernel<1><<<grid, kThreads, kSmemAlloc, st>>>(tmQ, tmK, a);
    score_merge_kernel<<<m.n_rows, merge_threads, 0, st>>>(m, R, c, partial, lse2);
    score_tc_kernel<2><<<grid, kThreads, kSmemAlloc, st>>>(tmQ, tmK, a);
  } else {
    const size_t sm1 = (size_t)(kTileKeys + R) * (d + 1) * sizeof(float);
    const size_t sm2 = sm1 + (size_t)R * sizeof(float);
    static std::once_flag attr_once;
    std::call_once(attr_once, [] {
      cudaFuncSetAttribute(score_f32_stats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
      cudaFuncSetAttribute(score_f32_colsum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
    });
    const float* q = static_cast<const float*>(qwin);
    const float* Kf = static_cast<const float*>(K);
    score_f32_stats_kernel<<<total_tiles, 128, sm1, st>>>(m, R, d, c, q, Kf, partial);
    score_merge_kernel<<<m.n_rows, merge_threads, 0, st>>>(m, R, c, partial, lse2);
    score_f32_colsum_kernel<<<total_tiles, 128, sm2, st>>>(m, R, d, c, q, Kf, lse2, s);
  }
  return cuda_status(cudaGetLastError());
}

}  // namespace kvc
