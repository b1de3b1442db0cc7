// ssd.cu -- the offline step before the decode path: the shared-basis spectral
// decomposition of one projection's experts and the choice of widths, on the GPU
// (BitsMoE study-note page, Methodology: first split, the SVD of the stacked
// expert matrices, W_cat = U S Phi^T with Phi the shared input basis and P = U S;
// second split, each column of an expert's block P_e normalised,
// W_e = sum_k a_{e,k} p_{e,k} phi_k^T with ||p_{e,k}|| = 1).
//
// W_cat stacks the E matrices W_e [d_out][d_in] vertically, (E d_out) x d_in, so
// Phi spans the input space.  Its right singular vectors and singular values are
// the eigenvectors and square-rooted eigenvalues of the d_in x d_in Gram matrix
// G = W_cat^T W_cat = sum_e W_e^T W_e, and P = U S = W_cat Phi.  The step is
// computed that way:
//   1. G = W_cat^T W_cat                       (fp32 GEMM, cuBLAS, no TF32)
//   2. G = V Lambda V^T                        (fp32 symmetric eigensolver, cuSOLVER)
//   3. Phi = the r eigenvectors of the largest eigenvalues, in descending order,
//      each with its sign fixed so that its entry of largest magnitude is
//      positive (the SVD leaves the sign free); also Phi^T in fp16 for the decode
//      path, and s_k = sqrt(max(lambda_k, 0))  (this file's kernels)
//   4. P = W_cat Phi                           (fp32 GEMM, cuBLAS)
//   5. a_{e,k} = ||P_e[:,k]||, p_{e,k} = P_e[:,k] / a_{e,k} (0 when a = 0),
//      written as the packer's amps [E][r] and comps [E][r][d_out]   (this file's kernels)
// cuBLAS and cuSOLVER are loaded on first use with dlopen, so the library loads
// (and its other calls work) on a machine without them.
#include <cublas_v2.h>
#include <cusolverDn.h>
#include <dlfcn.h>

#include <algorithm>
#include <mutex>
#include <thread>
#include <vector>

#include "common.cuh"

namespace bitsmoe {

// ---------------------------------------------------------------------------
// kernels
// ---------------------------------------------------------------------------
// One warp per output component k: eigenvector d_in - 1 - k of V (cuSOLVER's
// column-major eigenvectors, ascending eigenvalues; column j is row j of the
// row-major [d_in][d_in] array), sign-fixed, written as row k of Phi^T in fp32
// (for the GEMM) and fp16 (for the decode path), and s_k.
__global__ void k_ssd_phi(const float* __restrict__ V, const float* __restrict__ lambda, int d_in, int r,
                          float* __restrict__ phit32, uint16_t* __restrict__ phit16, float* __restrict__ sigma) {
    const int lane = threadIdx.x & 31;
    const int k = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
    if (k >= r) return;
    const int src = d_in - 1 - k;
    const float* v = V + (size_t)src * d_in;
    // the entry of largest magnitude (the first one on a tie)
    float best = -1.0f;
    int bi = 0x7fffffff;
    for (int i = lane; i < d_in; i += 32) {
        const float m = fabsf(v[i]);
        if (m > best) {
            best = m;
            bi = i;
        }
    }
    for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ob > best || (ob == best && oi < bi)) {
            best = ob;
            bi = oi;
        }
    }
    const float sgn = v[bi] < 0.0f ? -1.0f : 1.0f;
    for (int i = lane; i < d_in; i += 32) {
        const float x = sgn * v[i];
        phit32[(size_t)k * d_in + i] = x;
        phit16[(size_t)k * d_in + i] = __half_as_ushort(__float2half_rn(x));
    }
    if (lane == 0 && sigma) sigma[k] = sqrtf(fmaxf(lambda[src], 0.0f));
}

// a_{e,k} = ||P_e[:,k]||: one CTA per (expert, 32 components), lane = component,
// warps over the expert's rows of P [E d_out][r] (row-major; 128-byte row pieces).
__global__ void k_ssd_amps(const float* __restrict__ P, int d_out, int r, float* __restrict__ amps) {
    __shared__ float s_part[8][32];
    const int e = blockIdx.y, k0 = blockIdx.x * 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int k = k0 + lane;
    float acc = 0.0f;
    if (k < r)
        for (int i = warp; i < d_out; i += 8) {
            const float x = P[((size_t)e * d_out + i) * r + k];
            acc = fmaf(x, x, acc);
        }
    s_part[warp][lane] = acc;
    __syncthreads();
    if (warp == 0 && k < r) {
        float s = 0.0f;
        for (int w = 0; w < 8; w++) s += s_part[w][lane];
        amps[(size_t)e * r + k] = sqrtf(s);
    }
}

// comps[e][k][i] = P[e d_out + i][k] / a_{e,k}: 32 x 32 tiles transposed through
// shared memory (both the reads and the writes are 128-byte rows).
__global__ void k_ssd_comps(const float* __restrict__ P, const float* __restrict__ amps, int d_out, int r,
                            float* __restrict__ comps) {
    __shared__ float tile[32][33];
    const int e = blockIdx.z, i0 = blockIdx.y * 32, k0 = blockIdx.x * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 8 rows of threads
    for (int y = ty; y < 32; y += 8) {
        const int i = i0 + y, k = k0 + tx;
        tile[y][tx] = i < d_out && k < r ? P[((size_t)e * d_out + i) * r + k] : 0.0f;
    }
    __syncthreads();
    for (int y = ty; y < 32; y += 8) {
        const int k = k0 + y, i = i0 + tx;
        if (k < r && i < d_out) {
            const float a = amps[(size_t)e * r + k];
            comps[((size_t)e * r + k) * d_out + i] = a > 0.0f ? tile[tx][y] / a : 0.0f;
        }
    }
}

__global__ void k_ssd_info(const int* __restrict__ info, int32_t* status) {
    if (threadIdx.x == 0 && *info != 0) atomicOr(status, BITSMOE_ST_NOCONVERGE);
}

// ---------------------------------------------------------------------------
// cuBLAS and cuSOLVER, loaded on first use
// ---------------------------------------------------------------------------
struct LinAlg {
    bool ok = false;
    cublasStatus_t (*blas_create)(cublasHandle_t*);
    cublasStatus_t (*blas_set_stream)(cublasHandle_t, cudaStream_t);
    cublasStatus_t (*blas_set_math)(cublasHandle_t, cublasMath_t);
    cublasStatus_t (*sgemm)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int, const float*,
                            const float*, int, const float*, int, const float*, float*, int);
    cusolverStatus_t (*dn_create)(cusolverDnHandle_t*);
    cusolverStatus_t (*dn_set_stream)(cusolverDnHandle_t, cudaStream_t);
    cusolverStatus_t (*syevd_size)(cusolverDnHandle_t, cusolverEigMode_t, cublasFillMode_t, int, const float*, int,
                                   const float*, int*);
    cusolverStatus_t (*syevd)(cusolverDnHandle_t, cusolverEigMode_t, cublasFillMode_t, int, float*, int, float*,
                              float*, int, int*);
};

static std::mutex g_la_mu;
static LinAlg g_la;
static bool g_la_tried = false;

template <typename F>
static bool sym(void* lib, const char* name, F& out) {
    out = reinterpret_cast<F>(dlsym(lib, name));
    return out != nullptr;
}

static const LinAlg* linalg() {
    std::lock_guard<std::mutex> lock(g_la_mu);
    if (!g_la_tried) {
        g_la_tried = true;
        void* blas = dlopen("libcublas.so.12", RTLD_NOW | RTLD_LOCAL);
        if (!blas) blas = dlopen("/usr/local/cuda/lib64/libcublas.so.12", RTLD_NOW | RTLD_LOCAL);
        void* solver = dlopen("libcusolver.so.11", RTLD_NOW | RTLD_LOCAL);
        if (!solver) solver = dlopen("/usr/local/cuda/lib64/libcusolver.so.11", RTLD_NOW | RTLD_LOCAL);
        LinAlg L;
        L.ok = blas && solver && sym(blas, "cublasCreate_v2", L.blas_create) &&
               sym(blas, "cublasSetStream_v2", L.blas_set_stream) && sym(blas, "cublasSetMathMode", L.blas_set_math) &&
               sym(blas, "cublasSgemm_v2", L.sgemm) && sym(solver, "cusolverDnCreate", L.dn_create) &&
               sym(solver, "cusolverDnSetStream", L.dn_set_stream) &&
               sym(solver, "cusolverDnSsyevd_bufferSize", L.syevd_size) && sym(solver, "cusolverDnSsyevd", L.syevd);
        g_la = L;
    }
    return g_la.ok ? &g_la : nullptr;
}

// One cuBLAS and one cuSOLVER handle per device, created on first use.
struct Handles {
    cublasHandle_t blas = nullptr;
    cusolverDnHandle_t dn = nullptr;
};
constexpr int kSsdMaxDevices = 256;
static Handles g_handles[kSsdMaxDevices];

static bool handles(const LinAlg* L, Handles* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSsdMaxDevices) return false;
    std::lock_guard<std::mutex> lock(g_la_mu);
    Handles& h = g_handles[dev];
    if (!h.blas) {
        if (L->blas_create(&h.blas) != CUBLAS_STATUS_SUCCESS) return false;
        L->blas_set_math(h.blas, CUBLAS_PEDANTIC_MATH);  // plain fp32, no TF32
    }
    if (!h.dn && L->dn_create(&h.dn) != CUSOLVER_STATUS_SUCCESS) return false;
    *out = h;
    return true;
}

static bool ssd_dims_ok(int E, int d_out, int d_in, int r) {
    return E >= 1 && d_out >= 1 && d_in >= 1 && r >= 1 && r <= d_in && (int64_t)E * d_out < (1ll << 31) &&
           (int64_t)d_in * d_in < (1ll << 31);
}

// Workspace: G (then V) [d_in][d_in], lambda [d_in], Phi^T fp32 [r][d_in], P [E d_out][r],
// the eigensolver's info word and its work array.
struct SsdWS {
    float *G, *lambda, *phit, *P, *work;
    int* info;
    uint64_t used;
};
static SsdWS ssd_ws(int E, int d_out, int d_in, int r, int lwork, uint8_t* base) {
    SsdWS w{};
    uint64_t used = 0;
    auto take = [&](uint64_t bytes) -> void* {
        const uint64_t off = roundup(used, 256);
        used = off + bytes;
        return base ? base + off : nullptr;
    };
    w.G = (float*)take(4ull * d_in * d_in);
    w.lambda = (float*)take(4ull * d_in);
    w.phit = (float*)take(4ull * r * d_in);
    w.P = (float*)take(4ull * E * d_out * r);
    w.info = (int*)take(16);
    w.work = (float*)take(4ull * (uint64_t)std::max(lwork, 1));
    w.used = used;
    return w;
}

// The eigensolver's work-array length for an n x n matrix (the matrix and
// eigenvalue pointers only describe the call; nothing is read through them).
static int ssd_lwork(int d_in, const float* G, const float* lambda, int* lwork) {
    const LinAlg* L = linalg();
    if (!L) return set_cuda_error(cudaErrorSharedObjectInitFailed);
    Handles h;
    if (!handles(L, &h)) return set_cuda_error(cudaErrorInitializationError);
    if (L->syevd_size(h.dn, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, d_in, G, d_in, lambda, lwork) !=
        CUSOLVER_STATUS_SUCCESS)
        return set_cuda_error(cudaErrorUnknown);
    return BITSMOE_OK;
}

}  // namespace bitsmoe

using namespace bitsmoe;

BITSMOE_API uint64_t bitsmoe_ssd_workspace_bytes(int32_t E, int32_t d_out, int32_t d_in, int32_t r) {
    if (!ssd_dims_ok(E, d_out, d_in, r)) return 0;
    int lwork = 0;
    if (ssd_lwork(d_in, nullptr, nullptr, &lwork) != BITSMOE_OK) return 0;
    return ssd_ws(E, d_out, d_in, r, lwork, nullptr).used;
}

BITSMOE_API int bitsmoe_ssd_decompose(const float* W, int32_t E, int32_t d_out, int32_t d_in, int32_t r,
                                      uint16_t* phi_t, float* phi_t32, float* sigma, float* amps, float* comps,
                                      void* workspace, uint64_t workspace_bytes, int32_t* status, void* stream) {
    if (!ssd_dims_ok(E, d_out, d_in, r)) return BITSMOE_EINVAL;
    if (!W || !phi_t || !amps || !comps || !workspace) return BITSMOE_EINVAL;
    if ((uintptr_t)workspace % 256 || (uintptr_t)W % 4) return BITSMOE_EINVAL;
    // G and lambda sit at the same offsets whatever the work array's length
    const SsdWS w0 = ssd_ws(E, d_out, d_in, r, 1, (uint8_t*)workspace);
    int lwork = 0;
    int rc = ssd_lwork(d_in, w0.G, w0.lambda, &lwork);
    if (rc) return rc;
    SsdWS w = ssd_ws(E, d_out, d_in, r, lwork, (uint8_t*)workspace);
    if (workspace_bytes < w.used) return BITSMOE_ESIZE;
    const LinAlg* L = linalg();
    Handles h;
    if (!L || !handles(L, &h)) return set_cuda_error(cudaErrorInitializationError);
    cudaStream_t s = (cudaStream_t)stream;
    if (L->blas_set_stream(h.blas, s) != CUBLAS_STATUS_SUCCESS || L->dn_set_stream(h.dn, s) != CUSOLVER_STATUS_SUCCESS)
        return set_cuda_error(cudaErrorUnknown);
    const int N = E * d_out;
    const float one = 1.0f, zero = 0.0f;
    // 1. G = W_cat^T W_cat.  Row-major W [N][d_in] is the column-major d_in x N matrix A,
    //    and G = A A^T (column-major d_in x d_in, symmetric).
    if (L->sgemm(h.blas, CUBLAS_OP_N, CUBLAS_OP_T, d_in, d_in, N, &one, W, d_in, W, d_in, &zero, w.G, d_in) !=
        CUBLAS_STATUS_SUCCESS)
        return set_cuda_error(cudaErrorUnknown);
    // 2. eigenvalues (ascending) and eigenvectors (overwriting G, column-major)
    if (L->syevd(h.dn, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, d_in, w.G, d_in, w.lambda, w.work, lwork,
                 w.info) != CUSOLVER_STATUS_SUCCESS)
        return set_cuda_error(cudaErrorUnknown);
    // 3. Phi^T: the top r eigenvectors, descending, sign-fixed; s_k
    k_ssd_phi<<<(unsigned)((r * 32 + 255) / 256), 256, 0, s>>>(w.G, w.lambda, d_in, r, w.phit, phi_t, sigma);
    rc = check_launch();
    if (rc) return rc;
    if (phi_t32) {
        const cudaError_t e = cudaMemcpyAsync(phi_t32, w.phit, 4ull * r * d_in, cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return set_cuda_error(e);
    }
    // 4. P = W_cat Phi: the column-major r x N matrix Phi^T A, i.e. row-major P [N][r].
    //    Row-major Phi^T [r][d_in] is the column-major d_in x r matrix Phi.
    if (L->sgemm(h.blas, CUBLAS_OP_T, CUBLAS_OP_N, r, N, d_in, &one, w.phit, d_in, W, d_in, &zero, w.P, r) !=
        CUBLAS_STATUS_SUCCESS)
        return set_cuda_error(cudaErrorUnknown);
    // 5. a and unit p per expert
    k_ssd_amps<<<dim3((unsigned)((r + 31) / 32), (unsigned)E), 256, 0, s>>>(w.P, d_out, r, amps);
    rc = check_launch();
    if (rc) return rc;
    k_ssd_comps<<<dim3((unsigned)((r + 31) / 32), (unsigned)((d_out + 31) / 32), (unsigned)E), 256, 0, s>>>(
        w.P, amps, d_out, r, comps);
    rc = check_launch();
    if (rc) return rc;
    // the eigensolver's info word: not 0 when it did not converge (or met a non-finite value)
    if (status) {
        k_ssd_info<<<1, 32, 0, s>>>(w.info, status);
        rc = check_launch();
        if (rc) return rc;
    }
    return BITSMOE_OK;
}

// Widths by descending amplitude within each expert (ties: lower k first): the
// first count[0] components get width[0], the next count[1] width[1], and so on.
BITSMOE_API int bitsmoe_assign_widths(const float* amps_host, int32_t E, int32_t r, const uint8_t* widths_in_order,
                                      const int32_t* counts, int32_t n, uint8_t* widths_host) {
    if (!amps_host || !widths_in_order || !counts || !widths_host || E < 1 || r < 1 || n < 1) return BITSMOE_EINVAL;
    int64_t total = 0;
    for (int j = 0; j < n; j++) {
        if (counts[j] < 0 || !width_ok(widths_in_order[j])) return counts[j] < 0 ? BITSMOE_EINVAL : BITSMOE_EWIDTH;
        total += counts[j];
    }
    if (total != r) return BITSMOE_EINVAL;
    // experts are independent: split over host threads
    auto run = [&](int e0, int e1) {
        std::vector<int> order((size_t)r);
        for (int e = e0; e < e1; e++) {
            const float* a = amps_host + (size_t)e * r;
            for (int k = 0; k < r; k++) order[(size_t)k] = k;
            std::stable_sort(order.begin(), order.end(), [a](int x, int y) { return a[x] > a[y]; });
            int pos = 0;
            for (int j = 0; j < n; j++)
                for (int c = 0; c < counts[j]; c++)
                    widths_host[(size_t)e * r + order[(size_t)pos++]] = widths_in_order[j];
        }
    };
    const int nt = (int)std::min<int64_t>({(int64_t)std::max(1u, std::thread::hardware_concurrency()), 32, E});
    std::vector<std::thread> pool;
    for (int t = 1; t < nt; t++) pool.emplace_back(run, (int)((int64_t)E * t / nt), (int)((int64_t)E * (t + 1) / nt));
    run(0, (int)((int64_t)E / nt));
    for (auto& th : pool) th.join();
    return BITSMOE_OK;
}
