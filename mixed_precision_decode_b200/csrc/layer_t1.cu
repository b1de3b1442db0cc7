// layer_t1.cu -- fused single-token layer forward: both projections, one
// persistent launch (one CTA per SM).
//
// The method (BitsMoE study-note page, Methodology, first split; second
// split; Execution): z = Phi^T x is computed once per token and reused by the
// token's top-k experts; each expert evaluates its width-grouped bit planes
// bit-serially:  y_i = sum_b sum_j 2^j sum_{k in G_b} c_k bit_{k,j,i}
//                      - sum_b (2^b - 1)/2 sum_{k in G_b} c_k,  c_k = a_k s_k z_k.
//
// Design for B200 at one token: the step moves ~24 MB (Phi of both
// projections dominates) and has one grid-wide dependency (every expert row
// needs all of z).  So every CTA issues ALL of its HBM reads at launch --
// its slice of Phi rows by TMA bulk copies into shared memory, its slice of
// bit planes and per-component metadata by cp.async -- then computes its
// z rows, meets the other CTAs at a bounded grid barrier, and evaluates its
// (projection, slot, 32-row block) tasks from shared memory.  The bit-serial
// sum over 32 members of one plane word uses eight 16-entry subset-sum tables
// (one per nibble of members): one conflict-free shared-memory lookup per 4
// bits.  The routed sum is done by the last CTA to finish each row block, in
// slot order, so results do not depend on timing.
#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace bitsmoe {

#ifndef BITSMOE_T1_THREADS
#define BITSMOE_T1_THREADS 512
#endif
constexpr int kT1Threads = BITSMOE_T1_THREADS;  // threads per CTA of the fused kernel
constexpr int kT1Warps = kT1Threads / 32;
constexpr int kRB = 32;            // rows per task (one per lane)
constexpr int kMaxUnitsPerCta = 8;
constexpr int kPhiBars = 4;        // mbarriers over the Phi slice
constexpr long long kWaitLimitNs = 2000000000LL;  // bounded waits: 2 s, then BITSMOE_ST_TIMEOUT

struct T1Proj {
    const uint8_t* blob;
    const uint16_t* phi_t;
    float* Z;     // [r] or null
    float* Ye;    // [K][d_out] or null
    float* Ysum;  // [d_out]
};

struct T1Params {
    T1Proj proj[2];
    const uint16_t* x;
    const int32_t* ids;
    const float* gw;
    int32_t* status;
    unsigned long long* barrier;  // persistent, zero-initialised once
    uint32_t* rb_count;           // [2][n_rb], persistent, zero-initialised once
    float* zbuf;                  // [2][r]
    float* scratch;               // [2][K][d_pad]: g_j * y for the ordered combine
    int d_in, d_out, d_pad, r, K, E;
    int n_rb, n_tasks, G;
    int phi_rows;       // Phi rows per CTA (last CTA may have fewer)
    int tasks_max;      // tasks per CTA (upper bound)
    int pw_max;         // plane words per unit (upper bound over both blobs)
    int members_max;    // padded bit-plane members per unit (upper bound)
    int meta_max;       // metadata bytes per unit (upper bound)
    int n16_max;        // fp16 members per unit (upper bound)
    // shared-memory layout (byte offsets)
    uint32_t sm_x, sm_a, sm_planes, sm_meta, sm_end;
    uint32_t a_z, a_tab, a_part, a_c16, a_desc, a_cm;
};

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ long long globaltimer() {
    long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait on an mbarrier phase; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > kWaitLimitNs) return false;
    return true;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// 16-byte async copy global -> shared; src_bytes = 0 fills zeros without reading.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}
// Shared load at a 32-bit shared address plus a constant byte offset.  Not
// volatile, so the compiler may schedule it; its address always derives from a
// descriptor loaded after the barrier that publishes the tables.
template <int OFF>
__device__ __forceinline__ float lds_f32_imm(uint32_t addr) {
    float v;
    asm("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(OFF));
    return v;
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_add_release_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// ---------------------------------------------------------------------------
// per-unit description (one routed (projection, slot) pair)
// ---------------------------------------------------------------------------
struct UnitInfo {
    int p, j, e;                 // projection, slot, expert (-1 when the id is out of range)
    float g;                     // gate weight
    int n16;                     // fp16 members
    int pw;                      // plane words
    int ntab;                    // nibble tables (8 per 32-member word)
    uint32_t meta_off[kNumGroups];  // offsets of each group's metadata inside this unit's staging slot
    uint32_t np[kNumGroups];     // padded members
    uint32_t n[kNumGroups];      // members
    uint32_t pw0[kNumGroups];    // first plane word of the group (bit-plane groups)
    uint32_t tab0[kNumGroups];   // first table of the group
    uint64_t planes_off[kNumGroups];  // byte offset of the group's planes in the blob
    uint64_t w16_off;                 // byte offset of the fp16 rows in the blob
};

__device__ inline void unit_info(const T1Params& P, int u, UnitInfo& U) {
    U.p = u / P.K;
    U.j = u % P.K;
    int e = P.ids[U.j];
    U.e = (e >= 0 && e < P.E) ? e : -1;
    U.g = P.gw[U.j];
    U.n16 = U.pw = U.ntab = 0;
    uint32_t moff = 0, pw = 0, tab = 0;
    if (U.e < 0) {
        for (int g = 0; g < kNumGroups; g++) U.n[g] = U.np[g] = U.pw0[g] = U.tab0[g] = U.meta_off[g] = 0;
        U.w16_off = 0;
        return;
    }
    const uint8_t* blob = P.proj[U.p].blob;
    const DirEntry d = read_dir(blob, U.e);
    for (int g = 0; g < kNumGroups; g++) {
        const int b = group_width(g);
        U.n[g] = d.count[g];
        U.np[g] = (uint32_t)group_members_padded(b, d.count[g]);
        U.meta_off[g] = moff;
        U.pw0[g] = pw;
        U.tab0[g] = tab;
        const uint64_t gbase = d.base + d.goff[g];
        if (b == 16) {
            moff += 6 * U.np[g];
            U.w16_off = gbase + 6 * (uint64_t)U.np[g];
            U.planes_off[g] = 0;
        } else {
            moff += 8 * U.np[g];
            U.planes_off[g] = gbase + 8 * (uint64_t)U.np[g];
            pw += (uint32_t)b * (U.np[g] / 32);
            tab += U.np[g] / 4;
        }
    }
    U.n16 = (int)U.n[0];
    U.pw = (int)pw;
    U.ntab = (int)tab;
}

// Plane word q of a unit -> (group, bit plane, word).
__device__ __forceinline__ void decode_pw(const UnitInfo& U, int q, int& g, int& jb, int& w) {
    g = 1;
#pragma unroll
    for (int gg = 2; gg < kNumGroups; gg++)
        if ((uint32_t)q >= U.pw0[gg]) g = gg;
    const int W = (int)(U.np[g] / 32);
    const int rel = q - (int)U.pw0[g];
    jb = rel / W;
    w = rel - jb * W;
}

// Tasks [t0, t1) of a CTA.  With no more units than CTAs, every CTA works on
// one unit only (units get floor or ceil of G/U CTAs, each a contiguous range
// of the unit's row blocks), so each CTA builds one unit's tables; otherwise
// the task list is cut into G contiguous pieces.
__host__ __device__ inline void cta_tasks(const T1Params& P, int cta, int& t0, int& t1) {
    const int U = 2 * P.K;
    if (U <= P.G) {
        const int u = (int)(((long long)cta * U) / P.G);
        const int c0 = (int)(((long long)u * P.G + U - 1) / U), c1 = (int)(((long long)(u + 1) * P.G + U - 1) / U);
        const int n = c1 - c0, i = cta - c0;
        t0 = u * P.n_rb + (int)(((long long)i * P.n_rb) / n);
        t1 = u * P.n_rb + (int)(((long long)(i + 1) * P.n_rb) / n);
    } else {
        t0 = (int)(((long long)cta * P.n_tasks) / P.G);
        t1 = (int)(((long long)(cta + 1) * P.n_tasks) / P.G);
    }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
// A run is a maximal set of consecutive tasks of this CTA that share a unit;
// its staged plane words are laid out [plane word][rows of the run].
struct RunInfo {
    int ui;        // unit index inside the CTA
    int t_first;   // first task
    int nt;        // tasks in the run
    int rows;      // staged rows (nt * kRB, clamped to d_pad)
    uint32_t off;  // word offset of the run in the staging buffer
};
constexpr int kMaxRuns = kMaxUnitsPerCta;
constexpr int kRunTasks = 4;  // tasks evaluated together (one accumulator each)

__global__ void __launch_bounds__(kT1Threads, 1) k_layer_t1(const T1Params P) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t s_bar[kPhiBars + 1];  // Phi chunks, then planes + metadata
    __shared__ UnitInfo s_unit[kMaxUnitsPerCta];
    __shared__ RunInfo s_run[kMaxRuns];
    __shared__ int s_abort, s_nruns;
    __shared__ unsigned long long s_bar_base;
    __shared__ float s_zp;
    __shared__ float s_zpw[kT1Warps];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cta = blockIdx.x;
    int t0, t1;
    cta_tasks(P, cta, t0, t1);
    const int u_first = t0 / P.n_rb;
    const int u_last = t1 > t0 ? (t1 - 1) / P.n_rb : u_first - 1;
    const int nunits = u_last - u_first + 1;
    const int rows_total = 2 * P.r;
    const int row0 = (int)(((long long)cta * rows_total) / P.G);
    const int row1 = (int)(((long long)(cta + 1) * rows_total) / P.G);
    const int nrows = row1 - row0;
    const uint32_t row_bytes = (uint32_t)P.d_in * 2;

    uint16_t* s_x = reinterpret_cast<uint16_t*>(smem + P.sm_x);
    uint8_t* s_a = smem + P.sm_a;
    uint32_t* s_planes = reinterpret_cast<uint32_t*>(smem + P.sm_planes);
    uint8_t* s_meta = smem + P.sm_meta;

    // ---- phase 0: Phi rows and x first (they need nothing), by one thread ----
    if (tid == 0) {
        for (int i = 0; i <= kPhiBars; i++) mbar_init(&s_bar[i], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_abort = 0;
        s_bar_base = ld_relaxed_u64(P.barrier);
        for (int bi = 0; bi < kPhiBars; bi++) {
            const int ra = row0 + (nrows * bi) / kPhiBars, rbnd = row0 + (nrows * (bi + 1)) / kPhiBars;
            uint32_t bytes = (uint32_t)(rbnd - ra) * row_bytes + (bi == 0 ? row_bytes : 0);
            mbar_expect_tx(&s_bar[bi], bytes);
            if (bi == 0) bulk_g2s(s_x, P.x, row_bytes, &s_bar[0]);
            for (int rr = ra; rr < rbnd;) {  // rows are contiguous inside a projection
                const int p = rr / P.r, k = rr - p * P.r;
                const int n = min(rbnd - rr, P.r - k);
                bulk_g2s(s_a + (size_t)(rr - row0) * row_bytes, P.proj[p].phi_t + (size_t)k * P.d_in,
                         (uint32_t)n * row_bytes, &s_bar[bi]);
                rr += n;
            }
        }
    }
    // routed experts of this CTA's units (two dependent reads: ids, then the directory)
    if (warp == 1 && lane < nunits) unit_info(P, u_first + lane, s_unit[lane]);
    __syncthreads();  // s_unit ready

    // runs of this CTA's tasks (one thread)
    if (tid == 32) {
        int nr = 0;
        uint32_t off = 0;
        for (int t = t0; t < t1;) {
            const int ui = t / P.n_rb - u_first;
            const int te = min(t1, (ui + u_first + 1) * P.n_rb);
            while (t < te) {
                const int nt = min(kRunTasks, te - t);
                RunInfo R;
                R.ui = ui;
                R.t_first = t;
                R.nt = nt;
                R.rows = nt * kRB;
                R.off = off;
                const UnitInfo& U = s_unit[ui];
                off += (uint32_t)(U.e >= 0 ? U.pw : 0) * (uint32_t)(nt * kRB);
                s_run[nr++] = R;
                t += nt;
            }
        }
        s_nruns = nr;
        // bit planes (one copy per run, tile and group: the group's b x W x 32 words of a
        // 32-row tile are contiguous) and per-component metadata (one copy per group)
        uint32_t bytes = 0;
        for (int ri = 0; ri < nr; ri++) {
            const UnitInfo& U = s_unit[s_run[ri].ui];
            if (U.e >= 0) bytes += 128u * (uint32_t)U.pw * (uint32_t)s_run[ri].nt;
        }
        for (int ui = 0; ui < nunits; ui++) {
            const UnitInfo& U = s_unit[ui];
            if (U.e < 0) continue;
            for (int g = 0; g < kNumGroups; g++) bytes += (group_width(g) == 16 ? 6u : 8u) * U.np[g];
        }
        mbar_expect_tx(&s_bar[kPhiBars], bytes);
        for (int ri = 0; ri < nr; ri++) {
            const RunInfo& R = s_run[ri];
            const UnitInfo& U = s_unit[R.ui];
            if (U.e < 0) continue;
            const uint8_t* blob = P.proj[U.p].blob;
            const int tile0 = R.t_first % P.n_rb;
            for (int k = 0; k < R.nt; k++)
                for (int g = 1; g < kNumGroups; g++) {
                    if (U.n[g] == 0) continue;
                    const uint32_t gw = (uint32_t)group_width(g) * (U.np[g] / 32) * kRB;  // words per tile
                    bulk_g2s(s_planes + R.off + (size_t)k * U.pw * kRB + (size_t)U.pw0[g] * kRB,
                             blob + U.planes_off[g] + 4ull * gw * (uint64_t)(tile0 + k), 4u * gw, &s_bar[kPhiBars]);
                }
        }
        for (int ui = 0; ui < nunits; ui++) {
            const UnitInfo& U = s_unit[ui];
            if (U.e < 0) continue;
            const uint8_t* blob = P.proj[U.p].blob;
            const DirEntry d = read_dir(blob, U.e);
            for (int g = 0; g < kNumGroups; g++) {
                if (U.n[g] == 0) continue;
                bulk_g2s(s_meta + (size_t)ui * P.meta_max + U.meta_off[g], blob + d.base + d.goff[g],
                         (group_width(g) == 16 ? 6u : 8u) * U.np[g], &s_bar[kPhiBars]);
            }
        }
    }

    // ---- phase 1: z rows of this CTA on every warp but warp 1 (which issues the plane copies) ----
    // The grid barrier is split: thread 0 arrives as soon as the row warps are
    // done (named barrier 1), and waits only after that.  The counter is a
    // multiple of G whenever no launch is in flight (it starts at zero and every
    // launch adds exactly G), so the value read at start rounded down to a
    // multiple of G is this launch's base.
    if (warp != 1) {
        const int wv = warp == 0 ? kT1Warps - 2 : warp - 2;  // 0 .. kT1Warps-2
        constexpr int kRowWarps = kT1Warps - 1;
        bool ok = nrows == 0 || mbar_wait(&s_bar[0], 0);  // barrier 0 carries x
        for (int rl = wv; ok && rl < nrows; rl += kRowWarps) {
            int bi = 0;
            while (bi + 1 < kPhiBars && rl >= (nrows * (bi + 1)) / kPhiBars) bi++;
            if (!mbar_wait(&s_bar[bi], 0)) {
                ok = false;
                break;
            }
            const uint4* rowv = reinterpret_cast<const uint4*>(s_a + (size_t)rl * row_bytes);
            const uint4* xv = reinterpret_cast<const uint4*>(s_x);
            float acc = 0.0f;
            for (int i8 = lane; i8 < P.d_in / 8; i8 += 32) {
                const uint4 a = rowv[i8], b = xv[i8];
                const __half2* ha = reinterpret_cast<const __half2*>(&a);
                const __half2* hb = reinterpret_cast<const __half2*>(&b);
#pragma unroll
                for (int h = 0; h < 4; h++) {
                    const float2 fa = __half22float2(ha[h]), fb = __half22float2(hb[h]);
                    acc = fmaf(fa.x, fb.x, acc);
                    acc = fmaf(fa.y, fb.y, acc);
                }
            }
            acc = warp_sum(acc);
            if (lane == 0) {
                const int rr = row0 + rl, p = rr / P.r, k = rr - p * P.r;
                P.zbuf[rr] = acc;
                if (P.proj[p].Z) P.proj[p].Z[k] = acc;
            }
        }
        if (!ok) s_abort = 1;
        asm volatile("bar.sync 1, %0;" ::"n"(kRowWarps * 32) : "memory");
        if (tid == 0) {
            // every bulk copy of Phi into this CTA's shared memory has landed (bounded)
            for (int bi = 0; bi < kPhiBars; bi++)
                if (!mbar_wait(&s_bar[bi], 0)) s_abort = 1;
            red_add_release_u64(P.barrier, 1ull);  // arrive
        }
    }
    __syncthreads();  // warp 1 has issued its copies; s_run is visible

    // ---- grid barrier wait (bounded), then the planes ----
    if (tid == 0) {
        const unsigned long long G = (unsigned long long)P.G;
        const unsigned long long target = (s_bar_base / G + 1) * G;
        if (ld_acquire_u64(P.barrier) < target) {
            const long long tw = globaltimer();
            while (ld_acquire_u64(P.barrier) < target) {
                if (globaltimer() - tw > kWaitLimitNs) {
                    s_abort = 1;
                    break;
                }
            }
        }
        if (!mbar_wait(&s_bar[kPhiBars], 0)) s_abort = 1;  // planes and metadata
        if (s_abort && P.status) atomicOr(P.status, BITSMOE_ST_TIMEOUT);
    }
    __syncthreads();
    if (s_abort) return;

    // ---- phase 2: z of the needed projections, then the runs ----
    float* s_z = reinterpret_cast<float*>(s_a + P.a_z);
    // tables start on a 512-byte shared-memory boundary: one word's 8 tables are 512 B, so the
    // byte address of a word's tables has a zero low byte and a lookup can splice the entry
    // offset into it with one byte permute
    float* s_tab = reinterpret_cast<float*>(s_a + P.a_tab + ((512u - (smem_u32(s_a + P.a_tab) & 511u)) & 511u));
    float* s_part = reinterpret_cast<float*>(s_a + P.a_part);
    float* s_c16 = reinterpret_cast<float*>(s_a + P.a_c16);
    uint2* s_desc = reinterpret_cast<uint2*>(s_a + P.a_desc);
    float* s_cm = reinterpret_cast<float*>(s_a + P.a_cm);
    const uint32_t tab_sbase = smem_u32(s_tab);
    {
        bool need[2] = {false, false};
        for (int ui = 0; ui < nunits; ui++) need[s_unit[ui].p] = true;
        for (int p = 0; p < 2; p++)
            if (need[p])
                for (int i = tid; i < P.r; i += kT1Threads) s_z[p * P.r + i] = __ldcg(P.zbuf + p * P.r + i);
    }
    __syncthreads();
    int cur_unit = -1;
    const int nruns = s_nruns;
    for (int ri = 0; ri < nruns; ri++) {
        const RunInfo R = s_run[ri];
        const UnitInfo& U = s_unit[R.ui];
        if (R.ui != cur_unit && U.e >= 0) {
            __syncthreads();  // the previous unit's tables and descriptors are no longer read
            const uint8_t* meta = s_meta + (size_t)R.ui * P.meta_max;
            const float* z = s_z + U.p * P.r;
            float zp = 0.0f;
            // pass 1: c_k = a_k s_k z_k of every member (bit-plane groups, concatenated in
            // group order and padded: member m of table tb is 4 tb + (m % 4)), and the
            // zero-point partial sums.  Group fields are copied to registers first: the
            // stores below go to shared memory, where UnitInfo also lives.
            for (int g = 1; g < kNumGroups; g++) {
                const uint32_t np = U.np[g], n = U.n[g], m0 = 4 * U.tab0[g];
                if (np == 0) continue;
                const uint8_t* gm = meta + U.meta_off[g];
                const float* __restrict__ amp = reinterpret_cast<const float*>(gm + 4 * np);
                const uint16_t* __restrict__ scl = reinterpret_cast<const uint16_t*>(gm + 2 * np);
                const uint16_t* __restrict__ idx = reinterpret_cast<const uint16_t*>(gm);
                const float hr = 0.5f * (float)((1 << group_width(g)) - 1);
                for (uint32_t ml = tid; ml < np; ml += kT1Threads) {
                    float c = 0.0f;
                    if (ml < n) c = amp[ml] * __half2float(__ushort_as_half(scl[ml])) * z[idx[ml]];
                    s_cm[m0 + ml] = c;
                    zp += hr * c;
                }
            }
            __syncthreads();
            // pass 2: entry n of table tb = sum of c over the set bits of n (one entry per
            // thread and step; four steps' loads are issued before their stores)
            {
                const int nent = 16 * U.ntab;
                const float4* __restrict__ cm4 = reinterpret_cast<const float4*>(s_cm);
                float* __restrict__ tab = s_tab;
                const int n = tid & 15;  // kT1Threads is a multiple of 16: n is fixed per thread
                for (int en0 = tid; en0 < nent; en0 += 4 * kT1Threads) {
                    float4 c4[4];
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        const int en = en0 + u * kT1Threads;
                        c4[u] = en < nent ? cm4[en >> 4] : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        const int en = en0 + u * kT1Threads;
                        if (en < nent)
                            tab[en] = ((n & 1 ? c4[u].x : 0.0f) + (n & 2 ? c4[u].y : 0.0f)) +
                                      ((n & 4 ? c4[u].z : 0.0f) + (n & 8 ? c4[u].w : 0.0f));
                    }
                }
            }
            // plane-word descriptors: shared-memory byte offset of the word's 8 tables, weight 2^j
            for (int q = tid; q < U.pw; q += kT1Threads) {
                int g, jb, w;
                decode_pw(U, q, g, jb, w);
                s_desc[q] = make_uint2(tab_sbase + 64u * (U.tab0[g] + 8u * (uint32_t)w), __float_as_uint((float)(1u << jb)));
            }
            if (U.n16 > 0) {
                const uint8_t* gm = meta + U.meta_off[0];
                const uint16_t* idx = reinterpret_cast<const uint16_t*>(gm);
                const float* amp = reinterpret_cast<const float*>(gm + 2 * U.np[0]);
                for (int m = tid; m < U.n16; m += kT1Threads) s_c16[m] = amp[m] * z[idx[m]];
            }
            zp = warp_sum(zp);
            if (lane == 0) s_zpw[warp] = zp;
            __syncthreads();
            if (warp == 0) {
                float v = lane < kT1Warps ? s_zpw[lane] : 0.0f;
                v = warp_sum(v);
                if (lane == 0) s_zp = v;
            }
            __syncthreads();
            cur_unit = R.ui;
        }
        // every warp takes a share of the unit's plane words for all tasks of the run
        float acc[kRunTasks];
#pragma unroll
        for (int k = 0; k < kRunTasks; k++) acc[k] = 0.0f;
        if (U.e >= 0) {
            const int stride = U.pw * kRB;  // words between consecutive tasks (tiles) of the run
            const uint32_t* pl = s_planes + R.off + lane;
            for (int q = warp; q < U.pw; q += kT1Warps) {
                const uint2 d = s_desc[q];
                const float wt = __uint_as_float(d.y);
#pragma unroll
                for (int k = 0; k < kRunTasks; k++) {
                    if (k < R.nt) {
                        const uint32_t word = pl[k * stride + q * kRB];
                        // entry offsets (nibble x 4 bytes): even nibbles in the bytes of lo, odd in hi;
                        // table n of this word is at d.x + 64 n, entry e at + 4 e
                        const uint32_t lo = (word << 2) & 0x3C3C3C3Cu, hi = (word >> 2) & 0x3C3C3C3Cu;
                        float l[8];
                        l[0] = lds_f32_imm<0>(__byte_perm(lo, d.x, 0x7650u));
                        l[1] = lds_f32_imm<64>(__byte_perm(hi, d.x, 0x7650u));
                        l[2] = lds_f32_imm<128>(__byte_perm(lo, d.x, 0x7651u));
                        l[3] = lds_f32_imm<192>(__byte_perm(hi, d.x, 0x7651u));
                        l[4] = lds_f32_imm<256>(__byte_perm(lo, d.x, 0x7652u));
                        l[5] = lds_f32_imm<320>(__byte_perm(hi, d.x, 0x7652u));
                        l[6] = lds_f32_imm<384>(__byte_perm(lo, d.x, 0x7653u));
                        l[7] = lds_f32_imm<448>(__byte_perm(hi, d.x, 0x7653u));
                        const float sum = ((l[0] + l[1]) + (l[2] + l[3])) + ((l[4] + l[5]) + (l[6] + l[7]));
                        acc[k] = fmaf(sum, wt, acc[k]);
                    }
                }
            }
            if (U.n16 > 0) {
                const uint16_t* w16 = reinterpret_cast<const uint16_t*>(P.proj[U.p].blob + U.w16_off);
#pragma unroll
                for (int k = 0; k < kRunTasks; k++) {
                    const int row = ((R.t_first + k) % P.n_rb) * kRB + lane;
                    if (k < R.nt && row < P.d_out)
                        for (int m = warp; m < U.n16; m += kT1Warps)
                            acc[k] = fmaf(s_c16[m], __half2float(__ushort_as_half(w16[(size_t)m * P.d_pad + row])),
                                          acc[k]);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < kRunTasks; k++) s_part[(k * kT1Warps + warp) * kRB + lane] = acc[k];
        __syncthreads();
        if (warp < R.nt) {  // warp k reduces task k of the run
            const int k = warp, t = R.t_first + k, rb = t % P.n_rb, row = rb * kRB + lane;
            float y = 0.0f;
            if (U.e >= 0) {
#pragma unroll
                for (int w = 0; w < kT1Warps; w++) y += s_part[(k * kT1Warps + w) * kRB + lane];
                y -= s_zp;
            }
            if (row < P.d_out) {
                if (P.proj[U.p].Ye) P.proj[U.p].Ye[(size_t)U.j * P.d_out + row] = y;
                P.scratch[((size_t)U.p * P.K + U.j) * P.d_pad + row] = U.e >= 0 ? U.g * y : 0.0f;
            }
        }
        __syncthreads();
    }
    // ordered routed sum: every task of this CTA is published with one fence, its
    // row-block counters bumped together, and the last slot of a row block sums
    // the K weighted rows in slot order.
    __threadfence();
    __syncthreads();
    __shared__ uint32_t s_last[64];
    const int ntask = t1 - t0;
    for (int i = tid; i < ntask; i += kT1Threads) {
        const int t = t0 + i, p = (t / P.n_rb) / P.K, rb = t % P.n_rb;
        const uint32_t old = atomicAdd(&P.rb_count[p * P.n_rb + rb], 1u);
        s_last[i] = old == (uint32_t)(P.K - 1);
    }
    __syncthreads();
    __threadfence();
    for (int i = warp; i < ntask; i += kT1Warps) {
        if (!s_last[i]) continue;
        const int t = t0 + i, p = (t / P.n_rb) / P.K, rb = t % P.n_rb;
        const int row = rb * kRB + lane;
        if (row < P.d_out) {
            float s = 0.0f;
            for (int j = 0; j < P.K; j++) s += __ldcg(P.scratch + ((size_t)p * P.K + j) * P.d_pad + row);
            P.proj[p].Ysum[row] = s;
        }
        if (lane == 0) P.rb_count[p * P.n_rb + rb] = 0u;
    }
    if (tid == 0 && P.status) {
        for (int ui = 0; ui < nunits; ui++)
            if (s_unit[ui].e < 0) atomicOr(P.status, BITSMOE_ST_BADEXPERT);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct T1Layout {
    bool ok;
    T1Params P;
    uint64_t ws_reserved;  // persistent counters at the start of the workspace
    uint64_t ws_bytes;
    size_t smem;
};

static int g_num_sms = 0;
static int g_max_smem = 0;

static bool device_info() {
    if (g_num_sms > 0) return true;
    int dev;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&g_max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
    return true;
}

static void unit_bounds(const bitsmoe_plan* p, int& pw, int& members, int& meta, int& n16) {
    for (int e = 0; e < p->dims.n_experts; e++) {
        const uint32_t* c = p->counts + 8 * (size_t)e;
        int w = 0, m = 0, mb = 0;
        for (int g = 0; g < kNumGroups; g++) {
            const int b = group_width(g);
            const int np = (int)group_members_padded(b, c[g]);
            if (b == 16) {
                mb += 6 * np;
            } else {
                mb += 8 * np;
                m += np;
                w += b * (np / 32);
            }
        }
        pw = std::max(pw, w);
        members = std::max(members, m);
        meta = std::max(meta, mb);
        n16 = std::max(n16, (int)c[0]);
    }
}

static uint32_t align_up(uint64_t v, uint64_t a) { return (uint32_t)roundup(v, a); }

// Shapes and workspace of the fused path; ok = false when they do not fit.
static T1Layout t1_layout(const bitsmoe_plan* g, const bitsmoe_plan* u) {
    T1Layout L{};
    L.ok = false;
    if (!device_info()) return L;
    T1Params& P = L.P;
    P.d_in = g->dims.d_in;
    P.d_out = g->dims.d_out;
    P.d_pad = (int)g->d_pad;
    P.r = g->dims.rank;
    P.K = g->dims.top_k;
    P.E = g->dims.n_experts;
    if (u->dims.d_out != P.d_out || u->dims.rank != P.r) return L;
    P.G = g_num_sms;
    P.n_rb = (P.d_out + kRB - 1) / kRB;
    P.n_tasks = 2 * P.K * P.n_rb;
    P.phi_rows = (2 * P.r + P.G - 1) / P.G;
    P.tasks_max = 0;
    int units_max = 0;
    for (int c = 0; c < P.G; c++) {  // exact bounds of the partition the kernel uses
        int a, b;
        cta_tasks(P, c, a, b);
        P.tasks_max = std::max(P.tasks_max, b - a);
        if (b > a) units_max = std::max(units_max, (b - 1) / P.n_rb - a / P.n_rb + 1);
    }
    int pw = 0, members = 0, meta = 0, n16 = 0;
    unit_bounds(g, pw, members, meta, n16);
    unit_bounds(u, pw, members, meta, n16);
    P.pw_max = pw;
    P.members_max = members;
    P.meta_max = align_up(meta, 16);
    P.n16_max = n16;

    if (units_max > kMaxUnitsPerCta || P.tasks_max > 64 || P.d_in % 8 || P.d_in > 8192) return L;
    if (units_max + (P.tasks_max + kRunTasks - 1) / kRunTasks > kMaxRuns) return L;
    // shared memory
    const uint64_t phi_bytes = (uint64_t)P.phi_rows * P.d_in * 2;
    P.a_z = 0;
    P.a_tab = align_up(P.a_z + 8ull * P.r, 128);
    P.a_part = align_up(P.a_tab + 512 + 16ull * 4 * (members / 4), 16);  // + 512: tables realigned in the kernel
    P.a_c16 = align_up(P.a_part + 4ull * kRunTasks * kT1Warps * kRB, 16);
    P.a_desc = align_up(P.a_c16 + 4ull * n16, 16);
    P.a_cm = align_up(P.a_desc + 8ull * P.pw_max, 16);
    const uint64_t a_bytes = std::max<uint64_t>(phi_bytes, P.a_cm + 4ull * members);
    P.sm_x = 0;
    P.sm_a = align_up(P.sm_x + 2ull * P.d_in, 128);
    P.sm_planes = align_up(P.sm_a + a_bytes, 128);
    P.sm_meta = align_up(P.sm_planes + 4ull * kRB * P.pw_max * P.tasks_max, 128);
    P.sm_end = align_up(P.sm_meta + (uint64_t)P.meta_max * units_max, 128);
    L.smem = P.sm_end;
    const size_t static_smem = sizeof(uint64_t) * kPhiBars + sizeof(UnitInfo) * kMaxUnitsPerCta + 256;
    if (L.smem + static_smem > (size_t)g_max_smem) return L;
    // workspace: [barrier | rb_count] persistent at the head, then zbuf and scratch
    L.ws_reserved = roundup(256 + 4ull * 2 * P.n_rb, 256);
    uint64_t off = roundup(4ull * 2 * P.r, 256);
    off = roundup(off + 4ull * 2 * P.K * P.d_pad, 256);
    L.ws_bytes = off;  // bytes after the reserved head
    L.ok = true;
    return L;
}

// Bytes the fused path uses after the reserved head (0 when it does not apply).
uint64_t layer_fused_t1_workspace(const bitsmoe_plan* g, const bitsmoe_plan* u) {
    T1Layout L = t1_layout(g, u);
    return L.ok ? L.ws_bytes : 0;
}

// Bytes at the head of a layer workspace that hold the fused path's
// persistent counters (0 when it does not apply).
uint64_t layer_fused_t1_reserved(const bitsmoe_plan* g, const bitsmoe_plan* u) {
    T1Layout L = t1_layout(g, u);
    return L.ok ? L.ws_reserved : 0;
}

int layer_forward_fused_t1(const bitsmoe_proj_io** io, const uint16_t* X, const int32_t* ids, const float* gw,
                           void* workspace, uint64_t workspace_bytes, int32_t* status, cudaStream_t s, bool* used) {
    *used = false;
    T1Layout L = t1_layout(io[0]->plan, io[1]->plan);
    if (!L.ok || workspace_bytes < L.ws_reserved + L.ws_bytes) return BITSMOE_OK;
    T1Params P = L.P;
    for (int j = 0; j < 2; j++) {
        P.proj[j].blob = (const uint8_t*)io[j]->blob;
        P.proj[j].phi_t = io[j]->phi_t;
        P.proj[j].Z = io[j]->Z;
        P.proj[j].Ye = io[j]->Y_experts;
        P.proj[j].Ysum = io[j]->Y_sum;
    }
    P.x = X;
    P.ids = ids;
    P.gw = gw;
    P.status = status;
    uint8_t* ws = (uint8_t*)workspace;
    P.barrier = (unsigned long long*)ws;
    P.rb_count = (uint32_t*)(ws + 256);
    uint64_t off = L.ws_reserved;
    P.zbuf = (float*)(ws + off);
    off = roundup(off + 4ull * 2 * P.r, 256);
    P.scratch = (float*)(ws + off);

    cudaError_t e = cudaFuncSetAttribute(k_layer_t1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem);
    if (e != cudaSuccess) return set_cuda_error(e);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)P.G);
    cfg.blockDim = dim3(kT1Threads);
    cfg.dynamicSmemBytes = L.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_layer_t1, P);
    if (e != cudaSuccess) return set_cuda_error(e);
    *used = true;
    return BITSMOE_OK;
}

}  // namespace bitsmoe

// ---------------------------------------------------------------------------
// Single-token layer forward with library-owned scratch, for callers that
// cannot allocate device memory.  The scratch (the fused kernel's grid-barrier
// counter, row-block counters, z of both projections and the weighted rows of
// the routed sum) lives in one fixed static device array instead of a
// caller-provided workspace.
// ---------------------------------------------------------------------------
namespace bitsmoe {

constexpr uint64_t kNoAllocScratchBytes = 1ull << 20;  // 1 MiB, held by every GPU that loads the library
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 256;
static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[kNoAllocMaxDevices];

// Device address of the scratch array on the current device, looked up once
// per device.  (In host code the array's name is only a host-side handle.)
static int noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_cuda_error(e);
    if (dev < 0 || dev >= kNoAllocMaxDevices) return BITSMOE_EINVAL;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return set_cuda_error(e);
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return BITSMOE_OK;
}

}  // namespace bitsmoe

BITSMOE_API int bitsmoe_layer_forward_t1_noalloc(const bitsmoe_proj_io* gate, const bitsmoe_proj_io* up,
                                                 const uint16_t* X, const int32_t* topk_ids, const float* gate_w,
                                                 int32_t* status, void* stream) {
    using namespace bitsmoe;
    if (!gate || !up || !gate->plan || !up->plan || !X || !topk_ids || !gate_w) return BITSMOE_EINVAL;
    const bitsmoe_proj_io* io[2] = {gate, up};
    const bitsmoe_plan *pg = gate->plan, *pu = up->plan;
    if (pg->dims.d_in != pu->dims.d_in || pg->dims.top_k != pu->dims.top_k ||
        pg->dims.n_experts != pu->dims.n_experts || pg->dims.d_in % 8)
        return BITSMOE_EINVAL;
    for (int j = 0; j < 2; j++) {
        if (!io[j]->blob || !io[j]->phi_t || !io[j]->Y_sum) return BITSMOE_EINVAL;
        if ((uintptr_t)io[j]->blob % 16 || (uintptr_t)io[j]->phi_t % 16) return BITSMOE_EINVAL;
    }
    if ((uintptr_t)X % 16) return BITSMOE_EINVAL;
    // shapes the single-launch kernel cannot hold, or whose scratch exceeds the array
    const uint64_t head = layer_fused_t1_reserved(pg, pu);
    const uint64_t rest = layer_fused_t1_workspace(pg, pu);
    if (head == 0 || rest == 0 || head + rest > kNoAllocScratchBytes) return BITSMOE_ESIZE;
    void* scratch = nullptr;
    int rc = noalloc_scratch(&scratch);
    if (rc) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    // the counters must start at zero; the array keeps whatever the last call left
    cudaError_t e = cudaMemsetAsync(scratch, 0, head, s);
    if (e != cudaSuccess) return set_cuda_error(e);
    bool used = false;
    rc = layer_forward_fused_t1(io, X, topk_ids, gate_w, scratch, head + rest, status, s, &used);
    if (rc) return rc;
    return used ? BITSMOE_OK : BITSMOE_ESIZE;
}
