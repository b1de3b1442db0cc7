// proj_tc.cu -- z = Phi^T x for a batch of tokens on the 5th-generation tensor
// cores (BitsMoE study-note page, Methodology, first split: the shared
// projection is computed once per token and reused by every routed expert; for
// a batch of tokens it is a dense fp16 contraction Z[t][k] = sum_i PhiT[k][i] X[t][i]).
//
// One CTA computes a 128 (rows of Phi^T) x N (tokens, padded to 16) tile over
// one K slice; the 8 CTAs of a cluster take the 8 K slices of the same tile and
// add their fp32 partial tiles through distributed shared memory in rank order
// (deterministic, no workspace) by pushing rows into the owning rank's shared
// memory with remote stores.  Operands arrive by 2-D TMA tiles
// (cp.async.bulk.tensor, 64 K-elements x rows, 128-byte swizzle; tokens past T
// read as zeros), one stage of K = 64 per mbarrier, all stages of a round issued
// at once; one thread issues each stage's tcgen05.mma (kind::f16, fp32
// accumulation in tensor memory) as soon as that stage has landed, so the loads
// of later stages overlap the MMAs of earlier ones; tcgen05.commit signals an
// mbarrier and four warps read the accumulator back with tcgen05.ld.  The step
// is HBM-bound (64 flop per Phi byte at T = 64).
#include <cuda.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "tc_common.cuh"

namespace bitsmoe {

constexpr int kTcThreads = 128;       // 4 warps: one per 32-lane TMEM sub-partition
constexpr int kTcM = 128;             // rows of Phi^T per tile
constexpr int kTcK = 64;              // K per stage (4 MMAs of K = 16)
constexpr int kTcCluster = 8;         // K slices per tile
constexpr int kTcMaxStages = 4;       // stages resident at once
constexpr int kTcBulkCols = 32;       // token tiles up to this width reduce by bulk copies (measured: faster at 16, slower at 64)

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
    uint32_t recv_off;  // byte offset of the receive slices (bulk reduction)
};

__global__ void __launch_bounds__(kTcThreads, 1) k_proj_tc(const TcParams P, const __grid_constant__ CUtensorMap tmA,
                                                           const __grid_constant__ CUtensorMap tmB) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t s_mbar;               // the MMAs of a round are done
    __shared__ uint64_t s_lbar[kTcMaxStages];  // stage st of a round has landed
    __shared__ uint64_t s_rbar;                // this rank's 8 row slices have arrived (bulk reduction)
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
        for (int st = 0; st < kTcMaxStages; st++)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tc_smem(&s_lbar[st])));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tc_smem(&s_rbar)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (P.n_pad <= kTcBulkCols)  // armed before any remote copy can arrive (the cluster barrier below)
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tc_smem(&s_rbar)),
                         "r"((uint32_t)(kTcCluster * 16 * 4) * (uint32_t)P.n_pad)
                         : "memory");
        s_fail = 0;
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // This CTA's mbarriers are initialised: arrive now, wait only before the first
    // remote access below (a CTA of the cluster may start later than this one).
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    const uint32_t tmem = s_tmem;
    const uint32_t idesc = tc_idesc(kTcM, n_pad);

    const uint32_t a_bytes = kTcM * kTcK * 2, b_bytes = (uint32_t)n_pad * kTcK * 2;
    uint32_t round = 0;
    bool accumulate = false;
    for (int kc = kbeg; kc < kend; kc += kTcK * kTcMaxStages, round++) {
        const int nst = min(kTcMaxStages, (kend - kc) / kTcK);
        if (tid == 0) {
            // every stage of the round at once: A = rows m0.. of Phi^T, B = the token tile
            for (int st = 0; st < nst; st++) {
                const int k0 = kc + st * kTcK;
                const uint32_t a_s = sbase + (uint32_t)st * P.stage_bytes, b_s = a_s + a_bytes;
                const uint32_t lb = tc_smem(&s_lbar[st]);
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(lb), "r"(a_bytes + b_bytes)
                             : "memory");
                tc_tma2d(a_s, &tmA, k0, m0, lb);
                tc_tma2d(b_s, &tmB, k0, P.t_base, lb);
            }
            // each stage's MMAs as soon as it has landed (K = 16 per MMA: 32 B along the swizzled row)
            bool ok = true;
            for (int st = 0; st < nst && ok; st++) {
                const uint32_t a_s = sbase + (uint32_t)st * P.stage_bytes, b_s = a_s + a_bytes;
                if (!tc_wait(tc_smem(&s_lbar[st]), round & 1u)) {
                    ok = false;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
                for (int kk = 0; kk < kTcK / 16; kk++) {
                    const uint64_t ad = tc_desc_sw128(a_s + 32u * kk);
                    const uint64_t bd = tc_desc_sw128(b_s + 32u * kk);
                    const uint32_t acc = accumulate ? 1u : 0u;
                    asm volatile(
                        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
                        "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
                        : "memory");
                    accumulate = true;
                }
            }
            if (!ok) s_fail = 1;
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                         : "memory");
        }
        // the stage buffers are reused (and the accumulator read) only after these MMAs finished
        if (!tc_wait(mbar, round & 1u)) s_fail = 1;
        __syncthreads();
        if (s_fail) break;
    }
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

    // The 8 partial tiles of the cluster are added by the rank that owns the rows
    // (rank q owns rows [16 q, 16 q + 16)), in rank order (deterministic).  Each CTA
    // first writes its accumulator to shared memory, [row][ldp] fp32.
    float* part = reinterpret_cast<float*>(smem);
    const int row = 32 * warp + lane;
    const int n_valid = min(n_pad, P.T - P.t_base);
    const bool bulk = n_pad <= kTcBulkCols;
    const int ldp = bulk ? n_pad : n_pad + 4;  // bulk: rows contiguous; pull: 16-byte aligned, padded
    for (int c0 = 0; c0 < n_pad; c0 += 16) {
        uint32_t v[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(part + row * ldp + c0 + i) =
                make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]), __uint_as_float(v[i + 2]),
                            __uint_as_float(v[i + 3]));
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    if (bulk) {
        // Each rank's 16 rows (one contiguous 16 x n_pad block) go to that rank's
        // receive slice [this rank] by one bulk copy, completing on its mbarrier; no
        // cluster barrier: the receive slices are memory no one else uses.
        float* recv = reinterpret_cast<float*>(smem + P.recv_off);  // [source rank][16][n_pad]
        const uint32_t slice = 16u * (uint32_t)n_pad * 4u;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // this thread's writes -> the copies' reads
        // every CTA of the cluster has initialised (and armed) its receive mbarrier
        asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
        __syncthreads();  // the partial tile is written
        if (tid == 0) {
            for (uint32_t q = 0; q < kTcCluster; q++) {
                uint32_t dst, bar;
                asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                             : "=r"(dst)
                             : "r"(tc_smem(recv + (size_t)rank * 16 * n_pad)), "r"(q));
                asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(bar) : "r"(tc_smem(&s_rbar)), "r"(q));
                asm volatile(
                    "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                        dst),
                    "r"(tc_smem(part + (size_t)q * 16 * n_pad)), "r"(slice), "r"(bar)
                    : "memory");
            }
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // the sources are read
        }
        if (!tc_wait(tc_smem(&s_rbar), 0)) s_fail = 1;  // this rank's 8 slices have arrived
        for (int e = tid; e < 16 * n_valid; e += kTcThreads) {
            const int rr = e & 15, n = e >> 4;  // consecutive threads: consecutive rows of one token
            float sum = 0.0f;
#pragma unroll
            for (int q = 0; q < kTcCluster; q++) sum += recv[((size_t)q * 16 + rr) * n_pad + n];
            P.Z[(size_t)(P.t_base + n) * P.r + m0 + 16 * (int)rank + rr] = sum;
        }
    } else {
        asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");  // the start-up arrival
        asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
        // pull: 4 columns at a time, the 8 remote 16-byte loads of an element group
        // issued back to back (their latencies overlap), then added in rank order
        const int ngrp = (n_valid + 3) / 4;
        for (int e = tid; e < 16 * ngrp; e += kTcThreads) {
            const int rr = 16 * (int)rank + (e & 15), cg = e >> 4;
            const uint32_t local = tc_smem(part + rr * ldp + 4 * cg);
            float4 v[kTcCluster];
#pragma unroll
            for (int q = 0; q < kTcCluster; q++) {
                uint32_t remote;
                asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(q));
                asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                             : "=f"(v[q].x), "=f"(v[q].y), "=f"(v[q].z), "=f"(v[q].w)
                             : "r"(remote));
            }
            float4 sum = v[0];
#pragma unroll
            for (int q = 1; q < kTcCluster; q++) {
                sum.x += v[q].x;
                sum.y += v[q].y;
                sum.z += v[q].z;
                sum.w += v[q].w;
            }
            const float sv[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
            for (int j = 0; j < 4; j++)
                if (4 * cg + j < n_valid) P.Z[(size_t)(P.t_base + 4 * cg + j) * P.r + m0 + rr] = sv[j];
        }
    }
    // no CTA leaves while another may still read its shared memory (the pull)
    if (!bulk) asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (s_fail && tid == 0 && P.status) atomicOr(P.status, BITSMOE_ST_TIMEOUT);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
}

// Whether the tensor-core path takes these shapes.
bool proj_tc_supported(int T, int d_in, int r) {
    return T >= 8 && r % kTcM == 0 && d_in % (kTcK * kTcCluster) == 0;
}

// A 2-D fp16 tensor map over rows x d_in (row-major), boxes of 64 K-elements x
// box_rows rows in the 128-byte swizzle; rows past the end read as zeros.
int tc_tensor_map(CUtensorMap* map, const uint16_t* base, int d_in, int rows, int box_rows) {
    const cuuint64_t dims[2] = {(cuuint64_t)d_in, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)d_in * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kTcK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    // The driver function comes through the runtime's entry-point query, so the
    // library does not link libcuda (it loads on a machine without a GPU driver).
    using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static std::atomic<EncodeFn> s_encode{nullptr};
    EncodeFn encode = s_encode.load(std::memory_order_acquire);
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return set_cuda_error(e);
        if (q != cudaDriverEntryPointSuccess || !fn) return set_cuda_error(cudaErrorSymbolNotFound);
        encode = reinterpret_cast<EncodeFn>(fn);
        s_encode.store(encode, std::memory_order_release);
    }
    const CUresult rc = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (void*)base, dims, strides, box, estr,
                               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return rc == CUDA_SUCCESS ? BITSMOE_OK : set_cuda_error(cudaErrorInvalidValue);
}

int launch_proj_tc(const uint16_t* phi_t, const uint16_t* X, float* Z, int T, int d_in, int r, int32_t* status,
                   cudaStream_t s) {
    CUtensorMap tmA;
    int rc = tc_tensor_map(&tmA, phi_t, d_in, r, kTcM);
    if (rc) return rc;
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
        P.stage_bytes = (uint32_t)(kTcM * kTcK * 2 + P.n_pad * kTcK * 2);  // a multiple of 1024 (n_pad % 16 == 0)
        CUtensorMap tmB;
        rc = tc_tensor_map(&tmB, X, d_in, T, P.n_pad);
        if (rc) return rc;
        // stages (later the partial tile), then the receive slices of the bulk reduction
        const size_t tile_bytes = std::max<size_t>((size_t)kTcMaxStages * P.stage_bytes, (size_t)kTcM * (P.n_pad + 4) * 4);
        P.recv_off = (uint32_t)roundup(tile_bytes, 128);
        const size_t smem = P.recv_off + (P.n_pad <= kTcBulkCols ? (size_t)kTcCluster * 16 * P.n_pad * 4 : 0) + 1024;
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
        e = cudaLaunchKernelEx(&cfg, k_proj_tc, P, tmA, tmB);
        if (e != cudaSuccess) return set_cuda_error(e);
    }
    return BITSMOE_OK;
}

}  // namespace bitsmoe
