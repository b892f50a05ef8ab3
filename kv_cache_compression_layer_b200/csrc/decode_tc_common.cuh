// Constants and device helpers of the tensor-core decode kernel (decode_tc.cu,
// one persistent kernel over all rows).
#pragma once

#include "decode_common.cuh"

namespace kvc {
namespace {

constexpr int kTcSlots = 64;                    // slots per TMA tile
constexpr int kCH = 128;                        // slots per work item
constexpr int kGroups = 3;                      // consumer groups of four warps
constexpr int kGStages = 2;                     // TMA stages per group
constexpr int kStages = kGroups * kGStages;
constexpr int kWarps = 4 * kGroups;
constexpr int kThreads = 32 * kWarps;
constexpr int kQBytes = kTcMaxG * 128 * 2;      // staged query rows per stage (d <= 128): two 8-row boxes
constexpr int kPartO = 2 * kTcMaxG;             // offset of O in a partial (16-byte aligned)
constexpr int kOutUnit = 256;                   // output elements per output unit
constexpr int kRowsBatch = 32;                  // row constants held at once by a CTA's finish

__device__ __forceinline__ uint32_t swz(uint32_t tile, int slot, int dcol) {
  const int box = dcol >> 6, chunk = (dcol & 63) >> 3;
  return tile + box * (kTcSlots * 128) + slot * 128 + ((chunk ^ (slot & 7)) << 4);
}
// Column of (head g, column c) in a group's combine buffer: the 32 lanes of one
// atomic (8 heads x 4 column pairs) land in 32 different banks.
__device__ __forceinline__ int ogswz(int g, int c) { return c ^ ((g & 3) << 3) ^ (g >> 2); }

// The staged query rows: two 64-column boxes of 8 rows, 128-byte swizzled.
__device__ __forceinline__ uint32_t qswz(uint32_t qarea, int row, int dcol) {
  const int box = dcol >> 6, chunk = (dcol & 63) >> 3;
  return qarea + box * 1024 + row * 128 + ((chunk ^ (row & 7)) << 4);
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

}  // namespace
}  // namespace kvc
