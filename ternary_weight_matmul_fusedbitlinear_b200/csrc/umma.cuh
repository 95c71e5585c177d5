// Device helpers for tcgen05 (UMMA, tensor memory) kernels and their TMA-stored
// epilogues on sm_100a.
#pragma once

#include "tma.cuh"

namespace mmf {

// Instruction descriptor of tcgen05.mma kind::i8: D s32, A s8 (activation
// codes), B u8 (weight codes w+1), both K-major, shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc_i8(int M, int N) {
  return (2u << 4)            // D format s32
         | (1u << 7)          // A format s8
         | (0u << 10)         // B format u8
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// UMMA shared-memory descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);   // start address
  d |= (uint64_t)1 << 16;                       // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;             // stride byte offset: next 8-row group
  d |= (uint64_t)1 << 46;                       // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                       // layout: SWIZZLE_128B
  return d;
}

__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(smem_u32(src))
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_le1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Stage one 32-row x 32-column box of the output in shared memory, in the
// layout the output tensor map's swizzle expects (lane = row): 2-byte types use
// 64-byte rows with the 64B swizzle (16-byte chunk c of row r at c ^ ((r>>1)&3)),
// 4-byte types 128-byte rows with the 128B swizzle (chunk c at c ^ (r&7)).
__device__ __forceinline__ void stage_row(uint8_t* buf, int r, const float (&v)[32], bf16*) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[8 * c + 2 * i], v[8 * c + 2 * i + 1]);
    *reinterpret_cast<uint4*>(buf + r * 64 + ((c ^ ((r >> 1) & 3)) << 4)) = u;
  }
}
__device__ __forceinline__ void stage_row(uint8_t* buf, int r, const float (&v)[32], float*) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<float4*>(buf + r * 128 + ((c ^ (r & 7)) << 4)) =
        make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}
__device__ __forceinline__ void stage_row_i32(uint8_t* buf, int r, const uint32_t (&v)[32], int qs) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<int4*>(buf + r * 128 + ((c ^ (r & 7)) << 4)) =
        make_int4((int)v[4 * c] - qs, (int)v[4 * c + 1] - qs, (int)v[4 * c + 2] - qs, (int)v[4 * c + 3] - qs);
}

// Add the residual box that TMA placed in `buf` (same swizzled layout as the
// staged output) to this lane's row of outputs.
__device__ __forceinline__ void add_staged_row(const uint8_t* buf, int r, float (&v)[32], bf16*) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 u = *reinterpret_cast<const uint4*>(buf + r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[8 * c + 2 * i] += f.x;
      v[8 * c + 2 * i + 1] += f.y;
    }
  }
}
__device__ __forceinline__ void add_staged_row(const uint8_t* buf, int r, float (&v)[32], float*) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float4 f = *reinterpret_cast<const float4*>(buf + r * 128 + ((c ^ (r & 7)) << 4));
    v[4 * c] += f.x;
    v[4 * c + 1] += f.y;
    v[4 * c + 2] += f.z;
    v[4 * c + 3] += f.w;
  }
}

// SiLU with the hardware exponential and approximate reciprocal (a few ulp).
__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.0f + __expf(-z)); }


}  // namespace mmf
