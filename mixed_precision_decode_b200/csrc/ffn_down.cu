// ffn_down.cu -- the expert FFN after the gate and up projections: SiLU(gate) * up
// and a dense fp16 down projection per expert, summed over each token's routed
// slots with its gate weights.
//
// The BitsMoE study-note page (Methodology) decomposes the gate and up
// projections of an expert and stops there.  What follows them is the usual
// gated expert:
//   h[t][j][m] = SiLU(Yg[t][j][m]) * Yu[t][j][m],      SiLU(v) = v / (1 + e^-v)
//   out[t][i]  = sum_j g[t][j] sum_m Wd[e][i][m] h[t][j][m],      e = ids[t][j]
// with Wd [E][d_model][d_ff] fp16 (row i of expert e = the weights of output i).
// It is HBM-bound: every routed expert's d_model x d_ff weights are read once.
//
// Two paths.
//  * One token (k_down_t1): a CTA owns a block of output rows for all top_k
//    slots, so the slot-order sum stays inside the CTA.  Before it waits for the
//    kernel ahead of it (programmatic dependent launch) it asks L2 for its rows of
//    every routed expert with bulk prefetches -- the weights are known before the
//    gate/up outputs exist -- and each warp loads its first rows into registers.
//    After the wait it forms h for every slot in shared memory; a warp dots 4 rows
//    of one slot at a time, lanes on 16-byte chunks, with every load of a step in
//    flight before its arithmetic.
//  * Several tokens: tokens are grouped by expert (the library's routing groups),
//    one output row is written per routed (token, slot) and the slot-order sum is a
//    second kernel.  For d_out <= 2048 the rows come from the tensor cores
//    (k_down_tc, below); otherwise k_down_mt: a CTA owns (expert, 128 rows; 32 when
//    a row's h needs several staged column blocks) and reads those rows once for up
//    to 4 of the expert's tokens per pass, with h staged in shared memory; each
//    warp works on 4 rows x 4 tokens at a time, its first rows loaded before h.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "tc_common.cuh"

namespace bitsmoe {

int launch_route_ids(const int32_t* ids, int npairs, int E, const RouteWS& rw, int32_t* status, cudaStream_t s);
int launch_combine(const int32_t* ids, const float* gw, float* Ye, float* Ysum, int T, int K, int E, int d_out,
                   cudaStream_t s);

constexpr int kDnThreads = 512;  // single-token kernel: 16 warps
constexpr int kDnWarps = kDnThreads / 32;
constexpr int kDnMaxRows = 64;            // output rows per CTA, at most
constexpr int kDnRowBatch = 4;            // rows a warp works on at once
constexpr int kDnChunks = 3;              // 16-byte chunks of a row a lane loads per step
constexpr int kDnMaxK = 64;               // slots the single-token kernel takes
constexpr int kDnT1MaxFloats = 40960;     // top_k x d_ff of h in one CTA's shared memory (160 KB)
constexpr uint32_t kDnPrefetchMax = 1u << 20;  // bytes per bulk L2 prefetch

constexpr int kDmThreads = 256;  // multi-token kernel: 8 warps x 4 rows
constexpr int kDmWarps = kDmThreads / 32;
constexpr int kDmRowsPerWarp = 4;
constexpr int kDmRows = kDmWarps * kDmRowsPerWarp;
constexpr int kDmTok = 4;       // tokens of one expert per pass
constexpr int kDmCols = 2048;   // columns of h per staged block (kDmTok x 2048 fp32 = 32 KB)
constexpr int kDmChunks = 3;    // 16-byte chunks of a row a lane loads per step
constexpr int kDmBatches = 4;   // batches of 4 rows per warp when h of a whole row fits one block

// SiLU with the fast exponential and division intrinsics: relative error a few
// 1e-6 where |v| < 100, far inside the outputs' 2e-3 bound; e^-v overflows to Inf
// for v below about -88 and the quotient is then 0 (the limit).
__device__ __forceinline__ float silu(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

// Bulk prefetch of [p, p + bytes) into L2, in pieces of at most kDnPrefetchMax bytes;
// bytes and p are multiples of 16.
__device__ __forceinline__ void prefetch_l2(const void* p, uint64_t bytes) {
    const uint8_t* c = static_cast<const uint8_t*>(p);
    while (bytes > 0) {
        const uint32_t n = bytes < kDnPrefetchMax ? (uint32_t)bytes : kDnPrefetchMax;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(c), "r"(n) : "memory");
        c += n;
        bytes -= n;
    }
}

// 16 bytes of weights, read once: not kept in L1.
__device__ __forceinline__ uint4 ld_weights(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// acc += the dot product of 8 fp16 weights with h0 (weights 0..3) and h1 (4..7).
__device__ __forceinline__ float dot8(const uint4 w, const float4 h0, const float4 h1, float acc) {
    const float2 w01 = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
    const float2 w23 = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
    const float2 w45 = __half22float2(*reinterpret_cast<const __half2*>(&w.z));
    const float2 w67 = __half22float2(*reinterpret_cast<const __half2*>(&w.w));
    acc = fmaf(w01.x, h0.x, acc);
    acc = fmaf(w01.y, h0.y, acc);
    acc = fmaf(w23.x, h0.z, acc);
    acc = fmaf(w23.y, h0.w, acc);
    acc = fmaf(w45.x, h1.x, acc);
    acc = fmaf(w45.y, h1.y, acc);
    acc = fmaf(w67.x, h1.z, acc);
    acc = fmaf(w67.y, h1.w, acc);
    return acc;
}

__device__ __forceinline__ float4 silu_mul(const float4 g, const float4 u) {
    return make_float4(silu(g.x) * u.x, silu(g.y) * u.y, silu(g.z) * u.z, silu(g.w) * u.w);
}

// ---------------------------------------------------------------------------
// one token
// ---------------------------------------------------------------------------
struct DownT1Params {
    const uint16_t* w;   // [E][d_model][d_ff]
    const float* yg;     // [K][d_ff]
    const float* yu;     // [K][d_ff]
    const int32_t* ids;  // [K]
    const float* gw;     // [K]
    float* out;          // [d_model]
    int32_t* status;
    int E, K, d_model, d_ff, rows;  // rows: output rows per CTA
};

// Loads, for the kDnRowBatch rows from `row` of expert e (n_valid of them inside the
// matrix), the 16-byte chunks c0 + lane + 32 u (u < kDnChunks) into wv; rows or chunks
// past the end, and every chunk of an expert of -1, are zero.
__device__ __forceinline__ void load_rows(uint4 (&wv)[kDnRowBatch][kDnChunks], const DownT1Params& P, int e, int row,
                                          int n_valid, int c0, int nch, int lane) {
    const uint4* wr = reinterpret_cast<const uint4*>(P.w + ((size_t)(e < 0 ? 0 : e) * P.d_model + row) * P.d_ff);
#pragma unroll
    for (int a = 0; a < kDnRowBatch; a++)
#pragma unroll
        for (int u = 0; u < kDnChunks; u++) {
            const int c = c0 + lane + 32 * u;
            wv[a][u] = e >= 0 && a < n_valid && c < nch ? ld_weights(wr + (size_t)a * nch + c) : make_uint4(0, 0, 0, 0);
        }
}

// Shared memory: h as [slot][half][chunk] float4 (half 0 = columns 8c..8c+3 of
// chunk c, half 1 = 8c+4..8c+7, so that consecutive lanes read consecutive
// 16-byte words), then the (row, slot) dot products, then the slots' experts
// and gate weights.
__global__ void __launch_bounds__(kDnThreads) k_down_t1(const DownT1Params P) {
    extern __shared__ __align__(16) float dsm[];
    const int nch = P.d_ff / 8;
    float4* s_h = reinterpret_cast<float4*>(dsm);                         // [K][2][nch]
    float* s_dot = dsm + (size_t)P.K * P.d_ff;                            // [rows][K]
    int* s_e = reinterpret_cast<int*>(s_dot + (size_t)P.rows * P.K);     // [K]
    float* s_g = reinterpret_cast<float*>(s_e + P.K);                     // [K]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row0 = blockIdx.x * P.rows;
    const int nrows = min(P.rows, P.d_model - row0);
    const int nrb = (nrows + kDnRowBatch - 1) / kDnRowBatch;  // row batches per slot
    const int nbatch = P.K * nrb;

    // Before the wait, the weights: this CTA's rows of every routed expert (one
    // contiguous range per slot) are requested into L2, and each warp loads its first
    // batch of rows into registers.  The ids may still be being written by an earlier
    // kernel, so they only choose what to read here: after the wait they are read
    // again, and a batch whose expert changed is loaded again.
    if (tid < P.K && nrows > 0) {
        const int e = P.ids[tid];
        if (e >= 0 && e < P.E)
            prefetch_l2(P.w + ((size_t)e * P.d_model + row0) * P.d_ff, 2ull * nrows * P.d_ff);
    }
    uint4 wv[kDnRowBatch][kDnChunks];
    const bool first_fits = nch <= 32 * kDnChunks;  // a batch's rows fit one step: preload it
    int e_pre = -1;
    if (first_fits && warp < nbatch) {
        const int j = warp / nrb;
        e_pre = P.ids[j];
        if (e_pre < 0 || e_pre >= P.E) e_pre = -1;
        load_rows(wv, P, e_pre, row0 + (warp - j * nrb) * kDnRowBatch, nrows - (warp - j * nrb) * kDnRowBatch, 0,
                  nch, lane);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (nrows <= 0) return;

    if (tid < P.K) {
        const int e = P.ids[tid];
        const bool ok = e >= 0 && e < P.E;
        s_e[tid] = ok ? e : -1;
        s_g[tid] = P.gw[tid];
        if (!ok && blockIdx.x == 0 && P.status) atomicOr(P.status, BITSMOE_ST_BADEXPERT);
    }
    __syncthreads();
    // h of every slot (zero for a slot whose id is out of range)
    {
        const int per_slot = P.d_ff / 4;  // float4 per slot
        const float4* g4 = reinterpret_cast<const float4*>(P.yg);
        const float4* u4 = reinterpret_cast<const float4*>(P.yu);
        for (int v = tid; v < P.K * per_slot; v += kDnThreads) {
            const int j = v / per_slot, c4 = v - j * per_slot;
            float4 h = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (s_e[j] >= 0) h = silu_mul(g4[v], u4[v]);
            s_h[((size_t)j * 2 + (c4 & 1)) * nch + (c4 >> 1)] = h;
        }
    }
    __syncthreads();
    // A warp takes kDnRowBatch rows of one slot at a time and, per step, issues all
    // kDnRowBatch x kDnChunks 16-byte weight loads of a lane before any arithmetic (6 KB
    // per warp in flight); h of a chunk is read once for all of the batch's rows.
    for (int b = warp; b < nbatch; b += kDnWarps) {
        const int j = b / nrb, rb = (b - j * nrb) * kDnRowBatch;
        const int e = s_e[j];
        float acc[kDnRowBatch];
#pragma unroll
        for (int a = 0; a < kDnRowBatch; a++) acc[a] = 0.0f;
        if (e >= 0) {
            const float4* h0 = s_h + (size_t)j * 2 * nch;
            const float4* h1 = h0 + nch;
#pragma unroll 1
            for (int c0 = 0; c0 < nch; c0 += 32 * kDnChunks) {
                if (!(first_fits && b == warp && e == e_pre)) load_rows(wv, P, e, row0 + rb, nrows - rb, c0, nch, lane);
#pragma unroll
                for (int u = 0; u < kDnChunks; u++) {
                    const int c = c0 + lane + 32 * u;
                    if (c >= nch) break;
                    const float4 ha = h0[c], hb = h1[c];
#pragma unroll
                    for (int a = 0; a < kDnRowBatch; a++) acc[a] = dot8(wv[a][u], ha, hb, acc[a]);
                }
            }
        }
#pragma unroll
        for (int a = 0; a < kDnRowBatch; a++) {
            const float d = warp_sum(acc[a]);
            if (lane == 0 && rb + a < nrows) s_dot[(rb + a) * P.K + j] = d;
        }
    }
    __syncthreads();
    for (int r = tid; r < nrows; r += kDnThreads) {
        float y = 0.0f;
        for (int j = 0; j < P.K; j++)
            if (s_e[j] >= 0) y = fmaf(s_g[j], s_dot[r * P.K + j], y);
        P.out[row0 + r] = y;
    }
}

// ---------------------------------------------------------------------------
// several tokens, grouped by expert
// ---------------------------------------------------------------------------
struct DownMtParams {
    const uint16_t* w;  // [E][d_model][d_ff]
    const float* yg;    // [T*K][d_ff]
    const float* yu;    // [T*K][d_ff]
    RouteWS rw;         // routing groups (count, start, active, nactive, pairs)
    float* ydown;       // [T*K][d_model]
    int E, d_model, d_ff;
};

// Loads the 16-byte chunks c0 + lane + 32 v (v < kDmChunks, inside [0, nchb)) of the
// kDmRowsPerWarp rows from `row` (n_valid of them inside the matrix) of the row-major
// matrix at wr (row_chunks chunks a row); the rest are zero.
__device__ __forceinline__ void load_rows_mt(uint4 (&wv)[kDmRowsPerWarp][kDmChunks], const uint4* wr, size_t row_chunks,
                                             int row, int n_valid, int c0, int nchb, int lane) {
#pragma unroll
    for (int a = 0; a < kDmRowsPerWarp; a++)
#pragma unroll
        for (int v = 0; v < kDmChunks; v++) {
            const int c = c0 + lane + 32 * v;
            wv[a][v] = a < n_valid && c < nchb ? ld_weights(wr + (size_t)(row + a) * row_chunks + c)
                                               : make_uint4(0, 0, 0, 0);
        }
}

// One CTA per (routed expert, block of rows): 8 warps, each with `bpw` batches of 4
// rows (bpw = 4 when h of a whole row fits one staged column block, else 1).
__global__ void __launch_bounds__(kDmThreads) k_down_mt(const DownMtParams P) {
    __shared__ __align__(16) float4 s_h[kDmTok * kDmCols / 4];  // [token][half][chunk] of one column block
    __shared__ int s_pair[kDmTok];
    const int slot = blockIdx.x;
    if (slot >= *P.rw.nactive) return;
    const int e = P.rw.active[slot];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ncb = (P.d_ff + kDmCols - 1) / kDmCols;      // column blocks of h
    const int bpw = ncb == 1 ? kDmBatches : 1;              // row batches per warp
    const int rows_cta = kDmWarps * kDmRowsPerWarp * bpw;
    const int row0 = blockIdx.y * rows_cta;
    const int nrows = min(rows_cta, P.d_model - row0);
    if (nrows <= 0) return;
    const uint16_t* wblk = P.w + ((size_t)e * P.d_model + row0) * P.d_ff;  // this CTA's rows: one range
    if (tid == 0) prefetch_l2(wblk, 2ull * nrows * P.d_ff);
    const size_t row_chunks = (size_t)P.d_ff / 8;
    const uint4* w16 = reinterpret_cast<const uint4*>(wblk);
    // the first batch's first step, before the routing groups and h are read (the
    // weights depend on neither)
    uint4 wv[kDmRowsPerWarp][kDmChunks];
    const int wrow0 = warp * bpw * kDmRowsPerWarp;  // this warp's first row in the block
    load_rows_mt(wv, w16, row_chunks, wrow0, nrows - wrow0, 0, min(kDmCols, P.d_ff) / 8, lane);
    bool have_pre = true;
    const int p0 = P.rw.start[e], p1 = P.rw.start[e + 1];

    for (int pq = p0; pq < p1; pq += kDmTok) {
        const int nt = min(kDmTok, p1 - pq);
        if (tid < kDmTok) s_pair[tid] = tid < nt ? P.rw.pairs[pq + tid] : -1;
        for (int bi = 0; bi < bpw; bi++) {
            const int r0 = wrow0 + bi * kDmRowsPerWarp;  // this batch's first row in the block
            float acc[kDmRowsPerWarp][kDmTok];
#pragma unroll
            for (int a = 0; a < kDmRowsPerWarp; a++)
#pragma unroll
                for (int u = 0; u < kDmTok; u++) acc[a][u] = 0.0f;
            for (int cb = 0; cb < ncb; cb++) {
                const int ncols = min(kDmCols, P.d_ff - cb * kDmCols);
                const int nchb = ncols / 8;
                if (ncb > 1 || bi == 0) {  // h of this column block (once per token group when one block)
                    __syncthreads();  // s_pair is written; the previous block's h is no longer read
                    for (int v = tid; v < nt * (ncols / 4); v += kDmThreads) {
                        const int u = v / (ncols / 4), c4 = v - u * (ncols / 4);
                        const size_t src = (size_t)s_pair[u] * P.d_ff + (size_t)cb * kDmCols + 4 * c4;
                        const float4 g = *reinterpret_cast<const float4*>(P.yg + src);
                        const float4 up = *reinterpret_cast<const float4*>(P.yu + src);
                        s_h[((size_t)u * 2 + (c4 & 1)) * nchb + (c4 >> 1)] = silu_mul(g, up);
                    }
                    __syncthreads();
                }
                const uint4* wr = w16 + (size_t)cb * (kDmCols / 8);
#pragma unroll 1
                for (int c0 = 0; c0 < nchb; c0 += 32 * kDmChunks) {
                    if (have_pre)
                        have_pre = false;  // the rows loaded before the loop: first group, batch, block and step
                    else
                        load_rows_mt(wv, wr, row_chunks, r0, nrows - r0, c0, nchb, lane);
#pragma unroll
                    for (int v = 0; v < kDmChunks; v++) {
                        const int c = c0 + lane + 32 * v;
                        if (c >= nchb) break;
#pragma unroll
                        for (int u = 0; u < kDmTok; u++) {
                            if (u >= nt) break;
                            const float4 h0 = s_h[((size_t)u * 2) * nchb + c], h1 = s_h[((size_t)u * 2 + 1) * nchb + c];
#pragma unroll
                            for (int a = 0; a < kDmRowsPerWarp; a++) acc[a][u] = dot8(wv[a][v], h0, h1, acc[a][u]);
                        }
                    }
                }
            }
#pragma unroll
            for (int a = 0; a < kDmRowsPerWarp; a++)
#pragma unroll
                for (int u = 0; u < kDmTok; u++) {
                    const float d = warp_sum(acc[a][u]);
                    if (lane == 0 && u < nt && r0 + a < nrows)
                        P.ydown[(size_t)s_pair[u] * P.d_model + row0 + r0 + a] = d;
                }
        }
        __syncthreads();  // s_pair is read above before the next group rewrites it
    }
}

// ---------------------------------------------------------------------------
// several tokens on the tensor cores (d_out of the gate/up projections <= 2048)
// ---------------------------------------------------------------------------
// Per routed expert the down step is a dense contraction, out[pair][i] = sum_m
// Wd[e][i][m] h[pair][m], over the expert's few tokens: one CTA per (expert, 128
// rows) computes it with tcgen05.mma (kind::f16, fp32 accumulation in tensor
// memory).  A = 128 rows of Wd[e] (fp16, K-major as stored), streamed by 2-D TMA
// tiles of 64 K-elements through a ring of 4 stages.  B = 16 rows built in shared
// memory by the CTA: for up to 8 tokens of the expert, h / s_u split into an fp16
// high part (rows 0..7) and the fp16 rest (rows 8..15), so that the two columns
// of a token add up to the product with h to fp32 accuracy; s_u is a power of two
// that puts the token's largest |h| in [2^14, 2^15), inside fp16's range.
constexpr int kDcThreads = 128;   // 4 warps: tensor-memory lanes 0..127 = the tile's rows
constexpr int kDcM = 128;         // rows of an expert's down matrix per tile
constexpr int kDcK = 64;          // K per stage: one 128-byte swizzled row of fp16
constexpr int kDcStages = 4;      // ring of A stages
constexpr int kDcTok = 8;         // tokens per pass
constexpr int kDcN = 2 * kDcTok;  // B rows: high parts, then low parts
constexpr int kDcMaxDff = 2048;   // B of every K stage stays resident: 16 x 2048 x 2 = 64 KB
constexpr uint32_t kDcAStage = kDcM * kDcK * 2;  // 16 KB
constexpr uint32_t kDcBStage = kDcN * kDcK * 2;  // 2 KB
constexpr uint32_t kDcTmemCols = 32;             // the smallest allocation; N = 16 columns used

struct DownTcParams {
    const float* yg;  // [T*K][d_ff]
    const float* yu;  // [T*K][d_ff]
    RouteWS rw;       // routing groups
    float* ydown;     // [T*K][d_model]
    int32_t* status;
    int E, d_model, d_ff;
    int nst;  // K stages: ceil(d_ff / kDcK)
};

// The 8 values h[m], m = 8c .. 8c+7, of a routed pair (fp32).
__device__ __forceinline__ void h8_of(const DownTcParams& P, int pair, int c, float (&h)[8]) {
    const float4* g = reinterpret_cast<const float4*>(P.yg + (size_t)pair * P.d_ff) + 2 * c;
    const float4* u = reinterpret_cast<const float4*>(P.yu + (size_t)pair * P.d_ff) + 2 * c;
    const float4 ha = silu_mul(g[0], u[0]), hb = silu_mul(g[1], u[1]);
    h[0] = ha.x; h[1] = ha.y; h[2] = ha.z; h[3] = ha.w;
    h[4] = hb.x; h[5] = hb.y; h[6] = hb.z; h[7] = hb.w;
}

__global__ void __launch_bounds__(kDcThreads, 1) k_down_tc(const DownTcParams P, const __grid_constant__ CUtensorMap tmW) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t s_full[kDcStages];   // A stage landed
    __shared__ uint64_t s_empty[kDcStages];  // the MMAs that read an A stage are done
    __shared__ uint64_t s_done;              // the MMAs of a pass are done
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail;
    __shared__ int s_pair[kDcTok];
    __shared__ unsigned s_amax[kDcTok];  // largest |h| of each token, as fp32 bits
    __shared__ float s_scale[kDcTok];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slot = blockIdx.x;
    if (slot >= *P.rw.nactive) return;
    const int e = P.rw.active[slot];
    const int p0 = P.rw.start[e], p1 = P.rw.start[e + 1];
    const int m0 = blockIdx.y * kDcM;
    if (m0 >= P.d_model) return;
    const uint32_t sbase = (tc_smem(smem_raw) + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - tc_smem(smem_raw));
    const uint32_t a_base = sbase;                           // kDcStages x 16 KB
    const uint32_t b_base = sbase + kDcStages * kDcAStage;   // nst x 2 KB
    uint8_t* b_gen = smem + kDcStages * kDcAStage;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc_smem(&s_tmem)),
                     "r"(kDcTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (int b = 0; b < kDcStages; b++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tc_smem(&s_full[b])));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tc_smem(&s_empty[b])));
        }
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tc_smem(&s_done)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_fail = 0;
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = s_tmem;
    const uint32_t idesc = tc_idesc(kDcM, kDcN);
    const int npass = (p1 - p0 + kDcTok - 1) / kDcTok;
    const int G = npass * P.nst;                 // A stages streamed: every pass reads the whole tile
    const int row_y = e * P.d_model + m0;        // the tile's first row in the [E d_model][d_ff] map
    auto issue = [&](int q) {                    // A stage q into ring buffer q mod kDcStages
        const int buf = q % kDcStages;
        const uint32_t fb = tc_smem(&s_full[buf]);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(fb), "r"(kDcAStage) : "memory");
        tc_tma2d(a_base + (uint32_t)buf * kDcAStage, &tmW, (q % P.nst) * kDcK, row_y, fb);
    };
    if (tid == 0)
        for (int q = 0; q < min(kDcStages, G); q++) issue(q);

    const int nch = P.d_ff / 8;     // 16-byte chunks of h (8 fp16) per B row inside d_ff
    const int nchp = P.nst * 8;     // ... padded to whole stages
    for (int pass = 0; pass < npass; pass++) {
        const int pq = p0 + pass * kDcTok, nt = min(kDcTok, p1 - pq);
        if (tid < kDcTok) {
            s_pair[tid] = tid < nt ? P.rw.pairs[pq + tid] : -1;
            s_amax[tid] = 0u;
        }
        __syncthreads();
        // the largest |h| of each token (non-negative fp32 values order like their bits)
        for (int i = tid; i < nt * nch; i += kDcThreads) {
            const int u = i / nch, c = i - u * nch;
            float h[8];
            h8_of(P, s_pair[u], c, h);
            float m = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; j++) m = fmaxf(m, fabsf(h[j]));
            atomicMax(&s_amax[u], __float_as_uint(m));
        }
        __syncthreads();
        if (tid < kDcTok) {
            const float m = __uint_as_float(s_amax[tid]);
            // 2^(exponent of m - 14), kept inside [2^-100, 2^113] so that its reciprocal is finite
            s_scale[tid] = m > 0.0f && m <= 3.0e38f ? ldexpf(1.0f, max(ilogbf(m) - 14, -100)) : 1.0f;
        }
        __syncthreads();
        // B, both parts of every token (zeros for absent tokens and past d_ff), in the
        // 128-byte swizzle: 16-byte chunk ch of row r sits at chunk ch ^ (r mod 8)
        for (int i = tid; i < kDcTok * nchp; i += kDcThreads) {
            const int u = i / nchp, c = i - u * nchp;
            uint4 hi = make_uint4(0, 0, 0, 0), lo = make_uint4(0, 0, 0, 0);
            if (u < nt && c < nch) {
                float h[8];
                h8_of(P, s_pair[u], c, h);
                const float inv = 1.0f / s_scale[u];  // a power of two: exact
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const float v0 = h[2 * j] * inv, v1 = h[2 * j + 1] * inv;
                    const __half a0 = __float2half_rn(v0), a1 = __float2half_rn(v1);
                    const __half b0 = __float2half_rn(v0 - __half2float(a0)), b1 = __float2half_rn(v1 - __half2float(a1));
                    hw[j] = (uint32_t)__half_as_ushort(a0) | ((uint32_t)__half_as_ushort(a1) << 16);
                    lw[j] = (uint32_t)__half_as_ushort(b0) | ((uint32_t)__half_as_ushort(b1) << 16);
                }
                hi = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                lo = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
            const int st = c >> 3, ch = c & 7;
            uint8_t* stage = b_gen + (size_t)st * kDcBStage;
            *reinterpret_cast<uint4*>(stage + u * 128 + ((ch ^ u) << 4)) = hi;                // row u
            *reinterpret_cast<uint4*>(stage + 1024 + u * 128 + ((ch ^ u) << 4)) = lo;         // row 8 + u
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // B -> the tensor core's reads
        __syncthreads();
        if (tid == 0) {
            bool ok = true;
            for (int s = 0; s < P.nst; s++) {
                const int g = pass * P.nst + s, buf = g % kDcStages;
                if (!tc_wait(tc_smem(&s_full[buf]), (uint32_t)(g / kDcStages) & 1u)) {
                    ok = false;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t a_s = a_base + (uint32_t)buf * kDcAStage, b_s = b_base + (uint32_t)s * kDcBStage;
#pragma unroll
                for (int kk = 0; kk < kDcK / 16; kk++) {
                    const uint64_t ad = tc_desc_sw128(a_s + 32u * kk), bd = tc_desc_sw128(b_s + 32u * kk);
                    const uint32_t acc = (s > 0 || kk > 0) ? 1u : 0u;
                    asm volatile(
                        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
                        "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
                        : "memory");
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                 tc_smem(&s_empty[buf]))
                             : "memory");
                // refill the buffer of the stage before this one, whose MMAs were issued first
                const int q = g - 1 + kDcStages;
                if (g >= 1 && q < G) {
                    const int qb = (g - 1) % kDcStages;
                    if (!tc_wait(tc_smem(&s_empty[qb]), (uint32_t)((g - 1) / kDcStages) & 1u)) {
                        ok = false;
                        break;
                    }
                    issue(q);
                }
            }
            if (!ok) s_fail = 1;
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                             tc_smem(&s_done))
                         : "memory");
        }
        if (!tc_wait(tc_smem(&s_done), (uint32_t)pass & 1u)) s_fail = 1;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        uint32_t v[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(tmem + ((uint32_t)(32 * warp) << 16)));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        const int row = m0 + 32 * warp + lane;
        if (row < P.d_model && !s_fail) {
#pragma unroll
            for (int u = 0; u < kDcTok; u++)
                if (u < nt)
                    P.ydown[(size_t)s_pair[u] * P.d_model + row] =
                        (__uint_as_float(v[u]) + __uint_as_float(v[kDcTok + u])) * s_scale[u];
        }
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();  // B, the accumulator and s_pair are reused by the next pass
        if (s_fail) break;
    }
    if (s_fail && tid == 0 && P.status) atomicOr(P.status, BITSMOE_ST_TIMEOUT);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kDcTmemCols) : "memory");
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// Largest dynamic shared memory k_down_t1 has been granted on each device, so that
// a call (inside a stream capture too) asks the runtime again only when it needs more.
constexpr int kDnMaxDevices = 256;
static std::atomic<int> g_down_smem[kDnMaxDevices];

static cudaError_t grant_down_smem(int dev, int bytes) {
    const bool cached = dev >= 0 && dev < kDnMaxDevices;
    if (cached && g_down_smem[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(k_down_t1, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess || !cached) return e;
    int prev = g_down_smem[dev].load(std::memory_order_relaxed);
    while (prev < bytes && !g_down_smem[dev].compare_exchange_weak(prev, bytes)) {
    }
    return cudaSuccess;
}

static bool ffn_dims_ok(const bitsmoe_ffn_dims* d) {
    return d && d->d_model >= 1 && d->d_ff >= 8 && d->d_ff % 8 == 0 && d->n_experts >= 1 && d->top_k >= 1;
}

static bool ffn_single_token(const bitsmoe_ffn_dims* d, int T) {
    return T == 1 && d->top_k <= kDnMaxK && (int64_t)d->top_k * d->d_ff <= kDnT1MaxFloats;
}

struct FfnWS {
    RouteWS route;
    float* ydown;
    uint64_t used;
};

static FfnWS ffn_ws(const bitsmoe_ffn_dims* d, int T, uint8_t* base) {
    FfnWS w{};
    uint64_t used = 0;
    auto take = [&](uint64_t bytes) -> void* {
        const uint64_t off = roundup(used, 256);
        used = off + bytes;
        return base ? base + off : nullptr;
    };
    const int E = d->n_experts, K = d->top_k;
    w.route.count = (int32_t*)take(4ull * E);
    w.route.start = (int32_t*)take(4ull * (E + 1));
    w.route.active = (int32_t*)take(4ull * E);
    w.route.nactive = (int32_t*)take(4);
    w.route.pairs = (int32_t*)take(4ull * (uint64_t)T * K + 4);
    w.route.cvals = nullptr;
    w.route.zp = nullptr;
    w.route.ldc = 0;
    w.ydown = (float*)take(4ull * (uint64_t)T * K * d->d_model);
    w.used = used;
    return w;
}

}  // namespace bitsmoe

using namespace bitsmoe;

BITSMOE_API uint64_t bitsmoe_ffn_down_workspace_bytes(const bitsmoe_ffn_dims* dims, int32_t T) {
    if (!ffn_dims_ok(dims) || T < 0) return 0;
    if (T == 0 || ffn_single_token(dims, T)) return 0;
    return ffn_ws(dims, T, nullptr).used;
}

BITSMOE_API int bitsmoe_ffn_down_launches(const bitsmoe_ffn_dims* dims, int32_t T) {
    if (!ffn_dims_ok(dims) || T < 0) return BITSMOE_EINVAL;
    if (T == 0) return 0;
    return ffn_single_token(dims, T) ? 1 : 3;
}

BITSMOE_API int bitsmoe_ffn_down(const bitsmoe_ffn_dims* dims, const uint16_t* w_down, const float* Y_gate,
                                 const float* Y_up, const int32_t* topk_ids, const float* gate_w, int32_t T,
                                 float* out, void* workspace, uint64_t workspace_bytes, int32_t* status,
                                 void* stream) {
    if (!ffn_dims_ok(dims) || T < 0) return BITSMOE_EINVAL;
    if (T == 0) return BITSMOE_OK;
    if (!w_down || !Y_gate || !Y_up || !topk_ids || !gate_w || !out) return BITSMOE_EINVAL;
    if ((uintptr_t)w_down % 16 || (uintptr_t)Y_gate % 16 || (uintptr_t)Y_up % 16 || (uintptr_t)out % 4)
        return BITSMOE_EINVAL;
    const uint64_t need = bitsmoe_ffn_down_workspace_bytes(dims, T);
    if (need > 0 && (!workspace || (uintptr_t)workspace % 256)) return BITSMOE_EINVAL;
    if (workspace_bytes < need) return BITSMOE_ESIZE;
    cudaStream_t s = (cudaStream_t)stream;
    const int E = dims->n_experts, K = dims->top_k, d_model = dims->d_model, d_ff = dims->d_ff;

    if (ffn_single_token(dims, T)) {
        int dev = 0, sms = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return set_cuda_error(e);
        DownT1Params P{};
        P.w = w_down;
        P.yg = Y_gate;
        P.yu = Y_up;
        P.ids = topk_ids;
        P.gw = gate_w;
        P.out = out;
        P.status = status;
        P.E = E;
        P.K = K;
        P.d_model = d_model;
        P.d_ff = d_ff;
        // rows per CTA: one CTA per SM where the rows allow, at most kDnMaxRows
        P.rows = std::min(kDnMaxRows, std::max(1, (d_model + sms - 1) / std::max(1, sms)));
        const unsigned grid = (unsigned)((d_model + P.rows - 1) / P.rows);
        const size_t smem = 4ull * K * d_ff + 4ull * P.rows * K + 8ull * K;
        e = grant_down_smem(dev, (int)smem);
        if (e != cudaSuccess) return set_cuda_error(e);
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kDnThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        // Programmatic dependent launch: the weight prefetches run while the kernel
        // ahead (the layer call that wrote Y_gate / Y_up) finishes.  No CTA waits on
        // another, so nothing here needs its CTAs resident together.
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, k_down_t1, P);
        if (e != cudaSuccess) return set_cuda_error(e);
        return BITSMOE_OK;
    }

    FfnWS w = ffn_ws(dims, T, (uint8_t*)workspace);
    int rc = launch_route_ids(topk_ids, T * K, E, w.route, status, s);
    if (rc) return rc;
    const int slots = (int)std::min<int64_t>((int64_t)E, (int64_t)T * K);
    if (d_ff <= kDcMaxDff && (int64_t)E * d_model < (1ll << 31)) {
        // the tensor cores: a CTA per (expert, 128 rows)
        CUtensorMap tmW;
        rc = tc_tensor_map(&tmW, w_down, d_ff, E * d_model, kDcM);
        if (rc) return rc;
        DownTcParams P{};
        P.yg = Y_gate;
        P.yu = Y_up;
        P.rw = w.route;
        P.ydown = w.ydown;
        P.status = status;
        P.E = E;
        P.d_model = d_model;
        P.d_ff = d_ff;
        P.nst = (d_ff + kDcK - 1) / kDcK;
        const size_t smem = 1024 + (size_t)kDcStages * kDcAStage + (size_t)P.nst * kDcBStage;
        cudaError_t e = cudaFuncSetAttribute(k_down_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return set_cuda_error(e);
        dim3 grid((unsigned)slots, (unsigned)((d_model + kDcM - 1) / kDcM));
        k_down_tc<<<grid, kDcThreads, smem, s>>>(P, tmW);
    } else {
        DownMtParams P{};
        P.w = w_down;
        P.yg = Y_gate;
        P.yu = Y_up;
        P.rw = w.route;
        P.ydown = w.ydown;
        P.E = E;
        P.d_model = d_model;
        P.d_ff = d_ff;
        const int rows_cta = kDmRows * (d_ff <= kDmCols ? kDmBatches : 1);
        dim3 grid((unsigned)slots, (unsigned)((d_model + rows_cta - 1) / rows_cta));
        k_down_mt<<<grid, kDmThreads, 0, s>>>(P);
    }
    rc = check_launch();
    if (rc) return rc;
    return launch_combine(topk_ids, gate_w, w.ydown, out, T, K, E, d_model, s);
}
