// shared_proj.cu -- z = Phi^T x, once per token (BitsMoE study-note page,
// Methodology, first split: the projection does not depend on the expert and
// every expert selected for the token reuses it).
//
// Phi^T is [r][d_in] fp16 (row k = phi_k, K-major), X is [T][d_in] fp16.
// Batches of 8 or more tokens go to the tensor-core kernel (proj_tc.cu) when
// r is a multiple of 128 and d_in of 512.  Otherwise one warp owns one row of Phi^T; the row is read from HBM once, kept in
// registers, and dotted with every token of the batch (fp32 accumulation of
// exact fp16 x fp16 products).  This is an HBM stream over Phi.
#include "common.cuh"

namespace bitsmoe {

constexpr int kSPWarps = 8;

// acc + the products of 8 fp16 pairs: mixed-precision FMAs (fp16 operands, exact
// in fp32; fp32 addend), no fp16 value converted on its own.
__device__ __forceinline__ float dot8(uint4 a, uint4 b, float acc) {
    asm("{\n"
        " .reg .f16 a0, a1, a2, a3, a4, a5, a6, a7, b0, b1, b2, b3, b4, b5, b6, b7;\n"
        " mov.b32 {a0, a1}, %1;\n mov.b32 {a2, a3}, %2;\n mov.b32 {a4, a5}, %3;\n mov.b32 {a6, a7}, %4;\n"
        " mov.b32 {b0, b1}, %5;\n mov.b32 {b2, b3}, %6;\n mov.b32 {b4, b5}, %7;\n mov.b32 {b6, b7}, %8;\n"
        " fma.rn.f32.f16 %0, a0, b0, %0;\n fma.rn.f32.f16 %0, a1, b1, %0;\n"
        " fma.rn.f32.f16 %0, a2, b2, %0;\n fma.rn.f32.f16 %0, a3, b3, %0;\n"
        " fma.rn.f32.f16 %0, a4, b4, %0;\n fma.rn.f32.f16 %0, a5, b5, %0;\n"
        " fma.rn.f32.f16 %0, a6, b6, %0;\n fma.rn.f32.f16 %0, a7, b7, %0;\n"
        "}"
        : "+f"(acc)
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w));
    return acc;
}

// Rows of d_in up to kMaxChunks*256 halves stay in registers; longer rows loop.
constexpr int kMaxChunks = 16;  // 16 x 8 halves x 32 lanes = 4096

__global__ void __launch_bounds__(kSPWarps * 32) k_shared_proj(const uint16_t* __restrict__ phi_t,
                                                               const uint16_t* __restrict__ X, float* __restrict__ Z,
                                                               int T, int d_in, int r) {
    const int lane = threadIdx.x & 31;
    const int k = blockIdx.x * kSPWarps + (threadIdx.x >> 5);
    if (k >= r) return;
    const int n8 = d_in / 8;
    const uint4* row = reinterpret_cast<const uint4*>(phi_t + (uint64_t)k * d_in);
    if (n8 <= kMaxChunks * 32) {
        uint4 v[kMaxChunks];
#pragma unroll
        for (int c = 0; c < kMaxChunks; c++) {
            int i8 = lane + 32 * c;
            v[c] = i8 < n8 ? __ldcs(row + i8) : make_uint4(0, 0, 0, 0);
        }
        for (int t = 0; t < T; t++) {
            const uint4* xr = reinterpret_cast<const uint4*>(X + (uint64_t)t * d_in);
            float acc = 0.0f;
#pragma unroll
            for (int c = 0; c < kMaxChunks; c++) {
                int i8 = lane + 32 * c;
                if (i8 < n8) acc = dot8(v[c], __ldg(xr + i8), acc);
            }
            acc = warp_sum(acc);
            if (lane == 0) Z[(uint64_t)t * r + k] = acc;
        }
    } else {
        for (int t = 0; t < T; t++) {
            const uint4* xr = reinterpret_cast<const uint4*>(X + (uint64_t)t * d_in);
            float acc = 0.0f;
            for (int i8 = lane; i8 < n8; i8 += 32) acc = dot8(__ldg(row + i8), __ldg(xr + i8), acc);
            acc = warp_sum(acc);
            if (lane == 0) Z[(uint64_t)t * r + k] = acc;
        }
    }
}

bool proj_tc_supported(int T, int d_in, int r);
int launch_proj_tc(const uint16_t* phi_t, const uint16_t* X, float* Z, int T, int d_in, int r, int32_t* status,
                   cudaStream_t s);

// T >= 8 tokens on the tensor cores when the shapes allow it, else the GEMV.
int launch_shared_proj(const uint16_t* phi_t, const uint16_t* X, float* Z, int T, int d_in, int r,
                       cudaStream_t s) {
    if (T == 0) return BITSMOE_OK;
    if (proj_tc_supported(T, d_in, r)) return launch_proj_tc(phi_t, X, Z, T, d_in, r, nullptr, s);
    dim3 grid((unsigned)((r + kSPWarps - 1) / kSPWarps));
    k_shared_proj<<<grid, kSPWarps * 32, 0, s>>>(phi_t, X, Z, T, d_in, r);
    return check_launch();
}

}  // namespace bitsmoe

using namespace bitsmoe;

BITSMOE_API int bitsmoe_shared_proj(const uint16_t* phi_t, const uint16_t* X, float* Z, int32_t T, int32_t d_in,
                                    int32_t r, void* stream) {
    if (T < 0 || d_in < 8 || d_in % 8 || r < 1) return BITSMOE_EINVAL;
    if (T == 0) return BITSMOE_OK;
    if (!phi_t || !X || !Z) return BITSMOE_EINVAL;
    if ((uintptr_t)phi_t % 16 || (uintptr_t)X % 16) return BITSMOE_EINVAL;
    return launch_shared_proj(phi_t, X, Z, T, d_in, r, (cudaStream_t)stream);
}
