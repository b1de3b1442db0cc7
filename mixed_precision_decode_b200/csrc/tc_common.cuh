// tc_common.cuh -- helpers of the library's tcgen05 kernels (the shared projection
// and the FFN's down projection): shared-memory matrix and instruction descriptors,
// 2-D TMA tile loads and bounded mbarrier waits.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace bitsmoe {

constexpr long long kTcWaitNs = 2000000000LL;  // bounded waits: 2 s, then BITSMOE_ST_TIMEOUT

__device__ __forceinline__ uint32_t tc_smem(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Shared-memory matrix descriptor of a K-major operand in the 128-byte swizzled
// layout that a TMA tile of 64 fp16 K-elements per row writes: start address,
// leading byte offset (unused for this layout; 16 B), stride byte offset between
// 8-row groups (1024 B), descriptor version 1, layout type 2 (128-byte swizzle).
// A K step of 16 elements inside the 128-byte row advances the start by 32 B.
__device__ __forceinline__ uint64_t tc_desc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)(1024u >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator, fp16 A and B, both K-major.
__host__ __device__ constexpr uint32_t tc_idesc(int m, int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// 2-D TMA tile load into this CTA's shared memory alone, completing on an mbarrier.
__device__ __forceinline__ void tc_tma2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity) {
    long long t0;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    for (;;) {
        uint32_t ok;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
        long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        if (t - t0 > kTcWaitNs) return false;
    }
}


// A 2-D fp16 tensor map over rows x inner (row-major), boxes of 64 inner elements x
// box_rows rows in the 128-byte swizzle; rows past the end read as zeros.
int tc_tensor_map(CUtensorMap* map, const uint16_t* base, int inner, int rows, int box_rows);

}  // namespace bitsmoe
