// Tensor-core (tcgen05) and tensor-copy (TMA) helpers for sm_100a, used by
// the DFloat11 matrix product (lwc_gemm.cu).
//
// Operand layout. Both operands of one MMA are K-major tiles in shared
// memory with the 128-byte swizzle: a row holds 64 BF16 values (128 bytes),
// eight rows form a 1024-byte group, and inside a group the 16-byte chunk j
// of row r sits at chunk position j ^ (r % 8). Groups follow each other
// every 1024 bytes. Each tile starts on a 1024-byte boundary, so the swizzle
// (applied by the hardware to address bits 4-6 from bits 7-9) and the
// layout agree. This is the layout a tensor copy with 128-byte swizzle and a
// 64-element inner box writes, and the one the decoder writes by hand.
//
// Shared-memory matrix descriptor (64 bits), per the PTX ISA's tcgen05
// "matrix descriptor" format:
//   bits  0-13  start address >> 4
//   bits 16-29  leading-dimension byte offset >> 4 (unused by swizzled
//               K-major layouts; set to 1)
//   bits 32-45  stride-dimension byte offset >> 4 (1024 bytes between
//               8-row groups: 64)
//   bits 46-47  descriptor version (1 on sm_100)
//   bits 49-51  base offset (0: tiles are 1024-byte aligned)
//   bit  52     leading-dimension offset mode (0)
//   bits 61-63  swizzle mode (2 = 128-byte swizzle)
// One MMA consumes K = 16 (32 bytes of each row); the next 16 columns of
// the same tile start 32 bytes further, so the start address field grows by 2.
//
// Instruction descriptor (32 bits) of kind::f16, per the same document:
//   bits 4-5 accumulator format (1 = F32), bits 7-9 A format and bits 10-12
//   B format (1 = BF16), bit 15 / 16 A / B major (0 = K-major), bits 17-22
//   N >> 3, bits 24-28 M >> 4.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "lwc_device.cuh"

namespace lwc {
namespace umma {

constexpr uint32_t kSwizzleRowBytes = 128;     // one K-major row of 64 BF16
constexpr uint32_t kSwizzleGroupBytes = 1024;  // eight rows

__host__ __device__ constexpr uint64_t smem_desc_sw128(uint32_t smem_addr) {
    return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)(kSwizzleGroupBytes >> 4) << 32) |
           (1ull << 46) | (2ull << 61);
}

// BF16 x BF16 -> F32, both operands K-major, an M x N tile.
__host__ __device__ constexpr uint32_t instr_desc_bf16_f32(uint32_t M, uint32_t N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// Byte offset of element (row r, column c) of a swizzled K-major tile
// (c < 64): the layout described at the top of this file.
__host__ __device__ constexpr uint32_t sw128_offset(uint32_t r, uint32_t c) {
    return r * kSwizzleRowBytes + ((((c >> 3) ^ r) & 7u) << 4) + ((c & 7u) << 1);
}

// ---- tensor memory ------------------------------------------------------------

// Whole warp: allocates `cols` (a power of two >= 32) TMEM columns and
// writes their address to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dev::smem_u32(dst)),
                 "r"(cols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

// Whole warp: frees what tmem_alloc returned.
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---- MMA ----------------------------------------------------------------------

// One thread: D[tmem] (+)= A[smem] * B[smem]^T for the shape in idesc;
// accumulate = 0 overwrites D.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}

// One thread: the mbarrier at `bar` gets one arrival once every MMA this
// thread issued before has completed (their shared-memory reads included).
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     dev::smem_u32(bar))
                 : "memory");
}

// Whole warp: 16 consecutive 32-bit columns of the warp's 32 TMEM lanes
// (lane i of the warp reads lane base + i), then waits for the load.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

// ---- tensor copy --------------------------------------------------------------

// One thread: a 2-D tiled tensor copy (no multicast) of the box at
// (x, y) of the tensor map into shared memory at `dst`, completing on
// `bar`. x times the element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, int32_t x, int32_t y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dev::smem_u32(dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(dev::smem_u32(bar))
        : "memory");
}

}  // namespace umma
}  // namespace lwc
