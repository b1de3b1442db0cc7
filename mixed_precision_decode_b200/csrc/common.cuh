// common.cuh -- internal definitions shared by the library's CUDA sources.
//
// The packed format (v2) and the quantiser are specified in include/bitsmoe.h;
// this file is the library's own reading of that specification.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bitsmoe.h"

#define BITSMOE_API extern "C" __attribute__((visibility("default")))

namespace bitsmoe {

// Groups inside an expert, in storage order.
constexpr int kNumGroups = 7;
__host__ __device__ constexpr int group_width(int g) {
    return g == 0 ? 16 : g == 1 ? 8 : g == 2 ? 6 : g == 3 ? 4 : g == 4 ? 3 : g == 5 ? 2 : 1;
}
__host__ __device__ inline int group_of_width(int b) {
    switch (b) {
        case 16: return 0;
        case 8: return 1;
        case 6: return 2;
        case 4: return 3;
        case 3: return 4;
        case 2: return 5;
        case 1: return 6;
        default: return -1;  // width 0 or invalid
    }
}
__host__ __device__ inline bool width_ok(int b) {
    return b == 0 || b == 1 || b == 2 || b == 3 || b == 4 || b == 6 || b == 8 || b == 16;
}
__host__ __device__ constexpr uint64_t roundup(uint64_t v, uint64_t m) { return (v + m - 1) / m * m; }

constexpr uint32_t kMagic = 0x454F4D42u;  // "BMOE"
constexpr uint32_t kVersion = 2;
constexpr uint64_t kHeaderBytes = 64;
constexpr uint64_t kDirEntryBytes = 64;

// Members padded per group: 32 for bit-plane groups (one u32 word holds one
// bit plane of 32 members for one row), 8 for the fp16 group.
__host__ __device__ inline uint64_t group_members_padded(int b, uint64_t n) {
    return n == 0 ? 0 : (b == 16 ? roundup(n, 8) : roundup(n, 32));
}
__host__ __device__ inline uint64_t group_bytes(int b, uint64_t n, uint64_t d_pad) {
    if (n == 0) return 0;
    uint64_t np = group_members_padded(b, n);
    if (b == 16) return 6 * np + 2 * np * d_pad;
    return 8 * np + 4 * (uint64_t)b * (np / 32) * d_pad;
}

// Word index of plane word [plane j][word w][row i] inside a group's planes
// (rows fastest; W = words per plane, d_pad = padded rows).
__host__ __device__ inline uint64_t plane_word(uint32_t j, uint32_t w, uint32_t W, uint32_t d_pad, uint32_t i) {
    return ((uint64_t)j * W + w) * d_pad + i;
}

// Directory entry of one expert, decoded.
struct DirEntry {
    uint64_t base;          // byte offset of the expert's data in the blob
    uint32_t goff[kNumGroups];  // group offsets from base
    uint32_t count[kNumGroups]; // members per group
};

// Decodes the directory entry at d (global or shared memory).
__device__ inline DirEntry parse_dir(const uint8_t* d) {
    DirEntry r;
    r.base = *reinterpret_cast<const uint64_t*>(d);
    const uint32_t* go = reinterpret_cast<const uint32_t*>(d + 16);
    const uint16_t* ct = reinterpret_cast<const uint16_t*>(d + 44);
#pragma unroll
    for (int g = 0; g < kNumGroups; g++) {
        r.goff[g] = go[g];
        r.count[g] = ct[g];
    }
    return r;
}

__device__ inline DirEntry read_dir(const uint8_t* blob, int e) {
    return parse_dir(blob + kHeaderBytes + kDirEntryBytes * (uint64_t)e);
}

// Pointers into one group of width b (1..8).
struct QGroup {
    const uint16_t* idx;
    const uint16_t* scale;
    const float* amp;
    const uint32_t* planes;  // [b][W][d_pad]
    uint32_t n, np, W;
};
__device__ inline QGroup qgroup(const uint8_t* blob, const DirEntry& d, int g) {
    QGroup q;
    const uint8_t* G = blob + d.base + d.goff[g];
    q.n = d.count[g];
    q.np = (uint32_t)group_members_padded(group_width(g), q.n);
    q.W = q.np / 32;
    q.idx = reinterpret_cast<const uint16_t*>(G);
    q.scale = reinterpret_cast<const uint16_t*>(G + 2 * (uint64_t)q.np);
    q.amp = reinterpret_cast<const float*>(G + 4 * (uint64_t)q.np);
    q.planes = reinterpret_cast<const uint32_t*>(G + 8 * (uint64_t)q.np);
    return q;
}

// Pointers into the fp16 group.
struct HGroup {
    const uint16_t* idx;
    const float* amp;
    const uint16_t* w16;  // [np][d_pad]
    uint32_t n, np;
};
__device__ inline HGroup hgroup(const uint8_t* blob, const DirEntry& d) {
    HGroup h;
    const uint8_t* G = blob + d.base + d.goff[0];
    h.n = d.count[0];
    h.np = (uint32_t)group_members_padded(16, h.n);
    h.idx = reinterpret_cast<const uint16_t*>(G);
    h.amp = reinterpret_cast<const float*>(G + 2 * (uint64_t)h.np);
    h.w16 = reinterpret_cast<const uint16_t*>(G + 6 * (uint64_t)h.np);
    return h;
}

// The quantiser, exactly as specified: t = p / s and u = t + 2^(b-1) as two
// separately rounded IEEE fp32 operations, q = clamp(floor(u), 0, 2^b - 1).
__device__ __forceinline__ uint32_t quantise(float p, int b, uint16_t sh, int& st) {
    float s = __half2float(__ushort_as_half(sh));
    if (!isfinite(s) || s < 0.0f) {
        st |= BITSMOE_ST_BADSCALE;
        return 0;
    }
    if (s == 0.0f) return 0;
    if (!isfinite(p)) {
        st |= BITSMOE_ST_NONFINITE;
        return 0;
    }
    float t = __fdiv_rn(p, s);
    float u = __fadd_rn(t, (float)(1 << (b - 1)));
    float f = floorf(u);
    float qmax = (float)((1 << b) - 1);
    if (f < 0.0f) return 0;
    if (f > qmax) return (uint32_t)qmax;
    return (uint32_t)f;
}

// Bounds checks of the checked build (compiled with -DBITSMOE_CHECKED): an
// index i into a buffer of n elements (or a byte range ending at i) is checked
// before use; outside, BITSMOE_ST_BOUNDS is OR-ed into the status word and the
// caller skips the access.  In the normal build the check is the constant true.
#ifdef BITSMOE_CHECKED
__device__ __forceinline__ bool in_bounds(uint64_t i, uint64_t n, int32_t* status) {
    if (i < n) return true;
    if (status) atomicOr(status, BITSMOE_ST_BOUNDS);
    return false;
}
#else
__device__ __forceinline__ constexpr bool in_bounds(uint64_t, uint64_t, int32_t*) { return true; }
#endif

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace bitsmoe

// Host-side helpers (defined in host.cu).
namespace bitsmoe {
int set_cuda_error(cudaError_t e);  // records the text, returns BITSMOE_ECUDA
int check_launch();                 // cudaGetLastError -> 0 or ECUDA

// Routing groups of one call (in the caller's workspace).
struct RouteWS {
    int32_t* count;    // [E]   (reused as the scatter cursor)
    int32_t* start;    // [E+1] first pair of each expert in `pairs`
    int32_t* active;   // [E]   experts with at least one pair, ascending
    int32_t* nactive;  // [1]
    int32_t* pairs;    // [T*K] pair index t*K + j, grouped by expert
    float* cvals;      // [T*K][ldc] c of every member of each pair's expert (multi-token path)
    float* zp;         // [T*K] each pair's zero-point total
    uint32_t ldc;      // floats per c row
};
}  // namespace bitsmoe

// The plan object (host).
struct bitsmoe_plan {
    bitsmoe_dims dims;
    uint32_t d_pad;
    uint64_t blob_bytes;
    uint8_t* header;        // header + directory image, 64 + 64 E bytes
    uint64_t header_bytes;
    uint32_t* counts;       // [E][8], groups in storage order, [7] = width 0
    uint32_t max_items;     // max over experts of (n16 + sum of words of bit-plane groups)
    uint32_t max_members_padded;  // max over experts of the padded member count (all groups)
    uint32_t max_t1_items;  // max over experts of (words of bit-plane groups + fp16 octets)
};
