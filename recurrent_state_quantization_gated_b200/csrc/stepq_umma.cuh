// Fifth-generation tensor-core helpers for sm_100a: tensor-memory (TMEM) allocation, loads,
// stores and fences, shared-memory matrix descriptors, instruction descriptors and the single-thread
// tcgen05.mma issue of kind::f16 (bf16 operands, fp32 accumulate), cta_group::1.
//
// Operand layouts are the canonical no-swizzle "core matrix" layouts: a core matrix is 8 rows of
// 16 bytes (8 bf16), stored as 128 contiguous bytes. For an operand with R rows along M (or N) and
// Kd columns along K:
//   K-major : element (r, k) at ((r/8) * (Kd/8) + k/8) * 64 + (r%8) * 8 + k%8      (bf16 units)
//             leading-byte offset (next core matrix along K) 128 B, stride-byte offset (next
//             8-row group) Kd * 16 B; one K = 16 step advances the start address by 256 B.
//   MN-major: element (r, k) at ((k/8) * (R/8) + r/8) * 64 + (k%8) * 8 + r%8
//             leading-byte offset (next 8 k-rows) R * 16 B, stride-byte offset (next 8-element
//             group along M/N) 128 B; one K = 16 step advances the start address by R * 32 B.
// The accumulator of an M = 128 MMA occupies TMEM lanes 0-127 (lane = row) and N consecutive
// 32-bit columns; warp w of the CTA may read lanes 32 (w % 4) to 32 (w % 4) + 31 only.
#pragma once
#include <cstdint>

#include "stepq_device.cuh"

namespace stepq {
namespace umma {

__host__ __device__ constexpr int kmajor_off(int r, int k, int Kd) {
    return ((r >> 3) * (Kd >> 3) + (k >> 3)) * 64 + (r & 7) * 8 + (k & 7);
}
__host__ __device__ constexpr int mnmajor_off(int r, int k, int R) {
    return ((k >> 3) * (R >> 3) + (r >> 3)) * 64 + (k & 7) * 8 + (r & 7);
}

// Shared-memory matrix descriptor (no swizzle, sm_100 descriptor version 1, base offset 0).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    return d;
}
// Descriptor of K-step ks (16 bf16 along K) of a K-major operand with Kd columns.
__device__ __forceinline__ uint64_t desc_kmajor(const void* base, int ks, int Kd) {
    return smem_desc(smem_addr(base) + ks * 256u, 128u, static_cast<uint32_t>(Kd) * 16u);
}
// Descriptor of K-step ks of an MN-major operand with R rows along M (or N).
__device__ __forceinline__ uint64_t desc_mnmajor(const void* base, int ks, int R) {
    return smem_desc(smem_addr(base) + ks * static_cast<uint32_t>(R) * 32u, static_cast<uint32_t>(R) * 16u, 128u);
}

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 D, dense.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
           (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A * B^T, issued by one thread. accumulate = 0 overwrites D.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The mbarrier receives one arrival when every tcgen05 operation this thread issued before has
// completed (operand reads included).
__device__ __forceinline__ void commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}

// Executed by one whole warp; the TMEM base address is written to *slot.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
// Executed by the warp that allocated.
__device__ __forceinline__ void tmem_free(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Generic-proxy shared-memory writes become visible to the tensor core (async proxy).
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// TMEM loads (warp-collective; this thread's lane). Each helper issues its loads and the wait
// for them in one asm statement, so that no use of the loaded registers can be scheduled before
// the data has arrived.
#define STEPQ_R16(o) "=r"(r[o + 0]), "=r"(r[o + 1]), "=r"(r[o + 2]), "=r"(r[o + 3]), "=r"(r[o + 4]), "=r"(r[o + 5]), \
    "=r"(r[o + 6]), "=r"(r[o + 7]), "=r"(r[o + 8]), "=r"(r[o + 9]), "=r"(r[o + 10]), "=r"(r[o + 11]),           \
    "=r"(r[o + 12]), "=r"(r[o + 13]), "=r"(r[o + 14]), "=r"(r[o + 15])

// 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : STEPQ_R16(0)
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : STEPQ_R16(0), STEPQ_R16(16)
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 16 columns at each of two addresses.
__device__ __forceinline__ void tmem_ld16x2(uint32_t ta, uint32_t tb, float (&va)[16], float (&vb)[16]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%33];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : STEPQ_R16(0), STEPQ_R16(16)
        : "r"(ta), "r"(tb)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        va[i] = __uint_as_float(r[i]);
        vb[i] = __uint_as_float(r[16 + i]);
    }
}
#undef STEPQ_R16

// TMEM stores (warp-collective): 32 consecutive 32-bit columns of this thread's lane, followed by
// the wait for their completion.
#define STEPQ_S16(o) "r"(__float_as_uint(v[o + 0])), "r"(__float_as_uint(v[o + 1])), "r"(__float_as_uint(v[o + 2])), \
    "r"(__float_as_uint(v[o + 3])), "r"(__float_as_uint(v[o + 4])), "r"(__float_as_uint(v[o + 5])),                 \
    "r"(__float_as_uint(v[o + 6])), "r"(__float_as_uint(v[o + 7])), "r"(__float_as_uint(v[o + 8])),                 \
    "r"(__float_as_uint(v[o + 9])), "r"(__float_as_uint(v[o + 10])), "r"(__float_as_uint(v[o + 11])),               \
    "r"(__float_as_uint(v[o + 12])), "r"(__float_as_uint(v[o + 13])), "r"(__float_as_uint(v[o + 14])),              \
    "r"(__float_as_uint(v[o + 15]))
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        STEPQ_S16(0), STEPQ_S16(16)
        : "memory");
}
#undef STEPQ_S16

// TMEM address of (lane, column) relative to an allocation base.
__device__ __forceinline__ uint32_t tmem_at(uint32_t base, int lane, int col) {
    return base + (static_cast<uint32_t>(lane) << 16) + static_cast<uint32_t>(col);
}

}  // namespace umma
}  // namespace stepq
