// Device helpers shared by the kernels of the sparse+linear attention layer.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sla_internal.h"

namespace sla {

// ---------------------------------------------------------------------------
// device status word (lives at the start of the workspace)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void report(int* status, int code, int detail) {
  if (status == nullptr) return;
  if (atomicCAS(status, 0, code) == 0) status[1] = detail;
}

// ---------------------------------------------------------------------------
// conversions
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(v);
}

// elu(x) + 1
__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : __expf(x); }

// ---------------------------------------------------------------------------
// shared-memory addressing: rows of `rowbytes` bytes split in 16-byte chunks,
// chunk index XOR-ed with (row & 7) so that ldmatrix of 8 rows at one logical
// chunk touches 8 different bank groups.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t swz(int row, int chunk, int rowbytes) {
  return row * rowbytes + ((chunk ^ (row & 7)) << 4);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// cp.async (16 bytes, zero-fill when src_bytes == 0)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// ---------------------------------------------------------------------------
// ldmatrix / mma.sync (bf16, fp32 accumulate)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Lane addresses for ldmatrix.x4 of a 16x16 operand tile whose top-left is at
// (r0, c0) in a swizzled [rows][rowbytes] buffer; c0 counts 16-byte chunks.
//  A from [m][k] storage (non-trans): regs = a0..a3.
__device__ __forceinline__ uint32_t lds_a(uint32_t base, int r0, int ch0, int rowbytes, int lane) {
  return base + swz(r0 + (lane & 15), ch0 + (lane >> 4), rowbytes);
}
//  B from [n][k] storage (non-trans): regs = {b0,b1} of n-tile r0..r0+7, {b0,b1} of r0+8..r0+15.
__device__ __forceinline__ uint32_t lds_b_nk(uint32_t base, int r0, int ch0, int rowbytes, int lane) {
  return base + swz(r0 + (lane & 7) + ((lane >> 4) << 3), ch0 + ((lane >> 3) & 1), rowbytes);
}
//  B from [k][n] storage (trans): rows are k; regs = {b0,b1} of n-chunk ch0, {b0,b1} of ch0+1.
__device__ __forceinline__ uint32_t lds_b_kn(uint32_t base, int k0, int ch0, int rowbytes, int lane) {
  return base + swz(k0 + (lane & 7) + (((lane >> 3) & 1) << 3), ch0 + (lane >> 4), rowbytes);
}
//  A from [k][m] storage (trans): rows are k; regs = a0..a3 of m-chunk ch0 (16 rows of m).
__device__ __forceinline__ uint32_t lds_a_km(uint32_t base, int k0, int ch0, int rowbytes, int lane) {
  return base + swz(k0 + (lane & 7) + ((lane >> 4) << 3), ch0 + ((lane >> 3) & 1), rowbytes);
}

}  // namespace sla
