// proj_tc.cu -- z = Phi^T x for a batch of tokens on the 5th-generation tensor
// cores (BitsMoE study-note page, Methodology, first split: the shared
// projection is computed once per token and reused by every routed expert; for
// a batch of tokens it is a dense fp16 contraction Z[t][k] = sum_i PhiT[k][i] X[t][i]).
//
// One CTA computes a 128 (rows of Phi^T) x N (tokens, padded to 16) tile over
// one K slice; the 8 CTAs of a cluster take the 8 K slices of the same tile and
// add their fp32 partial tiles through distributed shared memory in rank order
// (deterministic, no workspace).  Operands are copied with cp.async into the
// canonical K-major no-swizzle layout (8-row x 16-byte core matrices), one
// thread issues tcgen05.mma (kind::f16, fp32 accumulation in tensor memory),
// tcgen05.commit signals an mbarrier, and four warps read the accumulator back
// with tcgen05.ld.  The step is HBM-bound (64 flop per Phi byte at T = 64).
#include <algorithm>

#include "common.cuh"

namespace bitsmoe {

constexpr int kTcThreads = 128;       // 4 warps: one per 32-lane TMEM sub-partition
constexpr int kTcM = 128;             // rows of Phi^T per tile
constexpr int kTcK = 64;              // K per stage (4 MMAs of K = 16)
constexpr int kTcCluster = 8;         // K slices per tile
constexpr int kTcMaxStages = 4;       // stages resident at once
constexpr long long kTcWaitNs = 2000000000LL;

struct TcParams {
    const uint16_t* phi_t;
    const uint16_t* X;
    float* Z;
    int32_t* status;
    int T, d_in, r;
    int n_pad;        // tokens of this launch's token tile, padded to a multiple of 16
    int t_base;       // first token of the tile
    int k_per_cta;    // K slice length (multiple of kTcK)
    uint32_t stage_bytes;
};

__device__ __forceinline__ uint32_t tc_smem(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Shared-memory matrix descriptor: start, leading (K-adjacent core matrices)
// and stride (M/N-adjacent 8-row groups) byte offsets, descriptor version 1,
// no swizzle.
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor, kind::f16: fp32 accumulator, fp16 A and B, both K-major.
__host__ __device__ constexpr uint32_t tc_idesc(int m, int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void tc_cp16(uint32_t dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
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

__global__ void __launch_bounds__(kTcThreads, 1) k_proj_tc(const TcParams P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t s_mbar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t rank;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    const int m0 = (blockIdx.x / kTcCluster) * kTcM;
    const int kbeg = (int)rank * P.k_per_cta, kend = kbeg + P.k_per_cta;
    const int n_pad = P.n_pad;
    const uint32_t ncols = n_pad <= 32 ? 32u : n_pad <= 64 ? 64u : n_pad <= 128 ? 128u : 256u;
    const uint32_t sbase = (tc_smem(smem_raw) + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - tc_smem(smem_raw));
    const uint32_t mbar = tc_smem(&s_mbar);

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc_smem(&s_tmem)),
                     "r"(ncols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mbar));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_fail = 0;
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = s_tmem;
    const uint32_t idesc = tc_idesc(kTcM, n_pad);

    uint32_t phase = 0;
    bool accumulate = false;
    for (int kc = kbeg; kc < kend && !s_fail; kc += kTcK * kTcMaxStages) {
        const int nst = min(kTcMaxStages, (kend - kc) / kTcK);
        // operands of nst stages into the K-major core-matrix layout (8 rows x 16 B per core matrix;
        // core matrix (row group i, K group j) at (8 i + j) * 128 bytes)
        for (int st = 0; st < nst; st++) {
            const int k0 = kc + st * kTcK;
            const uint32_t a_s = sbase + (uint32_t)st * P.stage_bytes, b_s = a_s + kTcM * kTcK * 2;
            for (int c = tid; c < kTcM * 8; c += kTcThreads) {
                const int rr = c >> 3, j = c & 7;
                tc_cp16(a_s + (uint32_t)(((rr >> 3) * 8 + j) * 128 + (rr & 7) * 16),
                        P.phi_t + (size_t)(m0 + rr) * P.d_in + k0 + 8 * j, 16u);
            }
            for (int c = tid; c < n_pad * 8; c += kTcThreads) {
                const int tt = c >> 3, j = c & 7;
                const int t = P.t_base + tt;
                const bool ok = t < P.T;
                tc_cp16(b_s + (uint32_t)(((tt >> 3) * 8 + j) * 128 + (tt & 7) * 16),
                        ok ? (const void*)(P.X + (size_t)t * P.d_in + k0 + 8 * j) : (const void*)P.X, ok ? 16u : 0u);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_all;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> tensor-core reads
        __syncthreads();
        if (tid == 0) {
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            for (int st = 0; st < nst; st++) {
                const uint32_t a_s = sbase + (uint32_t)st * P.stage_bytes, b_s = a_s + kTcM * kTcK * 2;
#pragma unroll
                for (int kk = 0; kk < kTcK / 16; kk++) {  // K = 16 per MMA: two core matrices along K
                    const uint64_t ad = tc_desc(a_s + 256u * kk, 128u, 1024u);
                    const uint64_t bd = tc_desc(b_s + 256u * kk, 128u, 1024u);
                    const uint32_t acc = accumulate ? 1u : 0u;
                    asm volatile(
                        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
                        "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
                        : "memory");
                    accumulate = true;
                }
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                         : "memory");
        }
        // the stage buffers are reused (and the accumulator read) only after these MMAs finished
        if (!tc_wait(mbar, phase)) s_fail = 1;
        phase ^= 1u;
        __syncthreads();
    }
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

    // partial tile -> shared memory [row][n_pad + 1] (padded rows: conflict-free)
    float* part = reinterpret_cast<float*>(smem);
    const int ldp = n_pad + 1;
    const int row = 32 * warp + lane;
    for (int c0 = 0; c0 < n_pad; c0 += 16) {
        uint32_t v[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int i = 0; i < 16; i++) part[row * ldp + c0 + i] = __uint_as_float(v[i]);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
    // rank q of the cluster adds the 8 partials of rows [16 q, 16 q + 16) in rank order
    const int n_valid = min(n_pad, P.T - P.t_base);
    for (int e = tid; e < 16 * n_valid; e += kTcThreads) {
        const int rr = 16 * (int)rank + (e & 15), n = e >> 4;
        const uint32_t local = tc_smem(part + rr * ldp + n);
        float s = 0.0f;
        for (uint32_t q = 0; q < kTcCluster; q++) {
            uint32_t remote;
            float v;
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(q));
            asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
            s += v;
        }
        P.Z[(size_t)(P.t_base + n) * P.r + m0 + rr] = s;
    }
    asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (s_fail && tid == 0 && P.status) atomicOr(P.status, BITSMOE_ST_TIMEOUT);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
}

// Whether the tensor-core path takes these shapes.
bool proj_tc_supported(int T, int d_in, int r) {
    return T >= 8 && r % kTcM == 0 && d_in % (kTcK * kTcCluster) == 0;
}

int launch_proj_tc(const uint16_t* phi_t, const uint16_t* X, float* Z, int T, int d_in, int r, int32_t* status,
                   cudaStream_t s) {
    for (int t_base = 0; t_base < T; t_base += 256) {
        TcParams P{};
        P.phi_t = phi_t;
        P.X = X;
        P.Z = Z;
        P.status = status;
        P.T = T;
        P.d_in = d_in;
        P.r = r;
        P.t_base = t_base;
        P.n_pad = (int)roundup((uint64_t)std::min(256, T - t_base), 16);
        P.k_per_cta = d_in / kTcCluster;
        P.stage_bytes = (uint32_t)(kTcM * kTcK * 2 + P.n_pad * kTcK * 2);
        const size_t smem = std::max<size_t>((size_t)kTcMaxStages * P.stage_bytes,
                                             (size_t)kTcM * (P.n_pad + 1) * 4) + 1024;
        cudaError_t e = cudaFuncSetAttribute(k_proj_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return set_cuda_error(e);
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)(r / kTcM * kTcCluster));
        cfg.blockDim = dim3(kTcThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kTcCluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, k_proj_tc, P);
        if (e != cudaSuccess) return set_cuda_error(e);
    }
    return BITSMOE_OK;
}

}  // namespace bitsmoe
