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

__device__ __forceinline__ float dot8(uint4 a, uint4 b, float acc) {
    const __half2* ha = reinterpret_cast<const __half2*>(&a);
    const __half2* hb = reinterpret_cast<const __half2*>(&b);
#pragma unroll
    for (int j = 0; j < 4; j++) {
        float2 fa = __half22float2(ha[j]);
        float2 fb = __half22float2(hb[j]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
    }
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
