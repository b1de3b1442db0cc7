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

constexpr int kT1Threads = 512;
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
    uint32_t a_z, a_tab, a_part, a_c16, a_desc;
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

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kT1Threads, 1) k_layer_t1(const T1Params P) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t s_bar[kPhiBars];
    __shared__ UnitInfo s_unit[kMaxUnitsPerCta];
    __shared__ int s_abort;
    __shared__ unsigned long long s_bar_base;
    __shared__ float s_zp;
    __shared__ float s_zpw[kT1Warps];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cta = blockIdx.x;
    const int t0 = (int)(((long long)cta * P.n_tasks) / P.G);
    const int t1 = (int)(((long long)(cta + 1) * P.n_tasks) / P.G);
    const int u_first = t0 / P.n_rb;
    const int u_last = t1 > t0 ? (t1 - 1) / P.n_rb : u_first - 1;
    const int rows_total = 2 * P.r;
    const int row0 = (int)(((long long)cta * rows_total) / P.G);
    const int row1 = (int)(((long long)(cta + 1) * rows_total) / P.G);
    const uint32_t row_bytes = (uint32_t)P.d_in * 2;

    uint16_t* s_x = reinterpret_cast<uint16_t*>(smem + P.sm_x);
    uint8_t* s_a = smem + P.sm_a;
    uint32_t* s_planes = reinterpret_cast<uint32_t*>(smem + P.sm_planes);
    uint8_t* s_meta = smem + P.sm_meta;

    // ---- phase 0: issue every HBM read: Phi rows and x first (they need nothing) ----
    if (tid == 0) {
        for (int i = 0; i < kPhiBars; i++) mbar_init(&s_bar[i], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_abort = 0;
        s_bar_base = ld_relaxed_u64(P.barrier);
        const int nrows = row1 - row0;
        for (int bi = 0; bi < kPhiBars; bi++) {
            const int ra = row0 + (nrows * bi) / kPhiBars, rbnd = row0 + (nrows * (bi + 1)) / kPhiBars;
            uint32_t bytes = (uint32_t)(rbnd - ra) * row_bytes + (bi == 0 ? row_bytes : 0);
            mbar_expect_tx(&s_bar[bi], bytes);
            if (bi == 0) bulk_g2s(s_x, P.x, row_bytes, &s_bar[0]);
            // rows [ra, rbnd) are contiguous inside each projection: at most two copies
            for (int rr = ra; rr < rbnd;) {
                const int p = rr / P.r, k = rr - p * P.r;
                const int n = min(rbnd - rr, P.r - k);
                bulk_g2s(s_a + (size_t)(rr - row0) * row_bytes, P.proj[p].phi_t + (size_t)k * P.d_in,
                         (uint32_t)n * row_bytes, &s_bar[bi]);
                rr += n;
            }
        }
    }
    // routed experts of this CTA's units (two dependent reads: ids, then the directory)
    if (tid >= 32 && tid - 32 < u_last - u_first + 1) unit_info(P, u_first + tid - 32, s_unit[tid - 32]);
    __syncthreads();

    // bit planes of this CTA's tasks: 32 rows x 4 B per plane word, 16 B per cp.async
    const int nunits = u_last - u_first + 1;
    for (int t = t0; t < t1; t++) {
        const UnitInfo& U = s_unit[t / P.n_rb - u_first];
        if (U.e < 0) continue;
        const int rb = t % P.n_rb;
        const uint8_t* blob = P.proj[U.p].blob;
        uint32_t* dst = s_planes + (size_t)(t - t0) * P.pw_max * kRB;
        for (int c = tid; c < U.pw * (kRB / 4); c += kT1Threads) {
            const int q = c / (kRB / 4), chunk = c % (kRB / 4);
            int g, jb, w;
            decode_pw(U, q, g, jb, w);
            const int row = rb * kRB + chunk * 4;
            const int W = (int)(U.np[g] / 32);
            const uint8_t* src = blob + U.planes_off[g] + 4 * (((uint64_t)jb * W + w) * P.d_pad + (uint64_t)row);
            const bool ok = row < P.d_pad;  // d_pad % 8 == 0: a 4-row chunk is all in or all out
            cp_async16(dst + (size_t)q * kRB + chunk * 4, ok ? src : blob, ok ? 16u : 0u);
        }
    }
    // per-component metadata (idx, scale, amp) of this CTA's units
    for (int ui = 0; ui < nunits; ui++) {
        const UnitInfo& U = s_unit[ui];
        if (U.e < 0) continue;
        const uint8_t* blob = P.proj[U.p].blob;
        const DirEntry d = read_dir(blob, U.e);
        for (int g = 0; g < kNumGroups; g++) {
            if (U.n[g] == 0) continue;
            const uint32_t bytes = (group_width(g) == 16 ? 6u : 8u) * U.np[g];
            const uint8_t* src = blob + d.base + d.goff[g];
            uint8_t* dst = s_meta + (size_t)ui * P.meta_max + U.meta_off[g];
            for (uint32_t o = (uint32_t)tid * 16; o < bytes; o += kT1Threads * 16) cp_async16(dst + o, src + o, 16);
        }
    }
    cp_async_commit();

    // ---- phase 1: z rows of this CTA ----
    {
        const int nrows = row1 - row0;
        bool ok = nrows == 0 || mbar_wait(&s_bar[0], 0);  // barrier 0 carries x
        for (int rl = warp; ok && rl < nrows; rl += kT1Warps) {
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
        // every bulk copy into this CTA's shared memory must have landed before it can exit
        if (tid == 0)
            for (int bi = 0; bi < kPhiBars; bi++)
                if (!mbar_wait(&s_bar[bi], 0)) s_abort = 1;
    }
    __syncthreads();

    // ---- grid barrier (bounded) ----
    // The counter is a multiple of G whenever no launch is in flight (it starts
    // at zero and every launch adds exactly G), so the value read at start
    // rounded down to a multiple of G is this launch's base.
    if (tid == 0) {
        const unsigned long long G = (unsigned long long)P.G;
        const unsigned long long target = (s_bar_base / G + 1) * G;
        red_add_release_u64(P.barrier, 1ull);
        if (ld_acquire_u64(P.barrier) < target) {
            const long long tw = globaltimer();
            while (ld_acquire_u64(P.barrier) < target) {
                if (globaltimer() - tw > kWaitLimitNs) {
                    s_abort = 1;
                    break;
                }
            }
        }
        if (s_abort && P.status) atomicOr(P.status, BITSMOE_ST_TIMEOUT);
    }
    __syncthreads();
    if (s_abort) {
        cp_async_wait_all();
        return;
    }

    // ---- phase 2: z of both projections into shared memory, then tasks ----
    float* s_z = reinterpret_cast<float*>(s_a + P.a_z);
    // tables must start on a 64-byte shared-memory boundary (lookups OR the entry offset into the base)
    float* s_tab = reinterpret_cast<float*>(s_a + P.a_tab + ((64u - (smem_u32(s_a + P.a_tab) & 63u)) & 63u));
    float* s_part = reinterpret_cast<float*>(s_a + P.a_part);
    float* s_c16 = reinterpret_cast<float*>(s_a + P.a_c16);
    for (int i = tid; i < 2 * P.r; i += kT1Threads) s_z[i] = __ldcg(P.zbuf + i);
    cp_async_wait_all();
    __syncthreads();

    uint2* s_desc = reinterpret_cast<uint2*>(s_a + P.a_desc);
    const uint32_t tab_sbase = smem_u32(s_tab);
    int cur_unit = -1;
    for (int t = t0; t < t1; t++) {
        const int ui = t / P.n_rb - u_first;
        const UnitInfo& U = s_unit[ui];
        const int rb = t % P.n_rb;
        const int row = rb * kRB + lane;
        if (ui != cur_unit && U.e >= 0) {
            __syncthreads();  // the previous unit's tables and descriptors are no longer read
            // nibble tables and the zero-point term of this unit
            const uint8_t* meta = s_meta + (size_t)ui * P.meta_max;
            const float* z = s_z + U.p * P.r;
            float zp = 0.0f;
            for (int tb = tid; tb < U.ntab; tb += kT1Threads) {
                int g = 1;
#pragma unroll
                for (int gg = 2; gg < kNumGroups; gg++)
                    if ((uint32_t)tb >= U.tab0[gg]) g = gg;
                const uint32_t np = U.np[g];
                const uint8_t* gm = meta + U.meta_off[g];
                const uint16_t* idx = reinterpret_cast<const uint16_t*>(gm);
                const uint16_t* scl = reinterpret_cast<const uint16_t*>(gm + 2 * np);
                const float* amp = reinterpret_cast<const float*>(gm + 4 * np);
                const uint32_t m0 = 4 * (tb - U.tab0[g]);
                float c[4];
#pragma unroll
                for (int b = 0; b < 4; b++) {
                    const uint32_t m = m0 + b;
                    c[b] = m < U.n[g] ? amp[m] * __half2float(__ushort_as_half(scl[m])) * z[idx[m]] : 0.0f;
                }
                float e[16];
                e[0] = 0.0f;
                e[1] = c[0];
                e[2] = c[1];
                e[3] = c[0] + c[1];
#pragma unroll
                for (int h = 0; h < 4; h++) e[4 + h] = e[h] + c[2];
#pragma unroll
                for (int h = 0; h < 8; h++) e[8 + h] = e[h] + c[3];
                float4* dst = reinterpret_cast<float4*>(s_tab + 16 * tb);
                dst[0] = make_float4(e[0], e[1], e[2], e[3]);
                dst[1] = make_float4(e[4], e[5], e[6], e[7]);
                dst[2] = make_float4(e[8], e[9], e[10], e[11]);
                dst[3] = make_float4(e[12], e[13], e[14], e[15]);
                zp += 0.5f * (float)((1 << group_width(g)) - 1) * ((c[0] + c[1]) + (c[2] + c[3]));
            }
            // plane-word descriptors: shared-memory byte offset of the word's 8 tables, weight 2^j
            for (int q = tid; q < U.pw; q += kT1Threads) {
                int g = 1;
#pragma unroll
                for (int gg = 2; gg < kNumGroups; gg++)
                    if ((uint32_t)q >= U.pw0[gg]) g = gg;
                const int W = (int)(U.np[g] / 32);
                const int rel = q - (int)U.pw0[g];
                const int jb = rel / W, w = rel - jb * W;
                s_desc[q] = make_uint2(tab_sbase + 64u * (U.tab0[g] + 8u * (uint32_t)w),
                                       __float_as_uint((float)(1u << jb)));
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
            if (tid == 0) {
                float sum = 0.0f;
                for (int w = 0; w < kT1Warps; w++) sum += s_zpw[w];
                s_zp = sum;
            }
            __syncthreads();
            cur_unit = ui;
        }
        float acc = 0.0f;
        if (U.e >= 0) {
            const uint32_t* pl = s_planes + (size_t)(t - t0) * P.pw_max * kRB + lane;
            for (int q = warp; q < U.pw; q += kT1Warps) {
                const uint2 d = s_desc[q];
                const uint32_t word = pl[q * kRB];
                // table t of this word sits at d.x + 64 t (64-byte aligned), entry n at + 4 n
                float l[8];
#pragma unroll
                for (int n = 0; n < 8; n++) {
                    const uint32_t off = n == 0 ? ((word << 2) & 0x3Cu) : ((word >> (4 * n - 2)) & 0x3Cu);
                    l[n] = lds_f32((d.x | off) + 64u * n);
                }
                const float sum = ((l[0] + l[1]) + (l[2] + l[3])) + ((l[4] + l[5]) + (l[6] + l[7]));
                acc = fmaf(sum, __uint_as_float(d.y), acc);
            }
            if (U.n16 > 0 && row < P.d_out) {
                const uint16_t* w16 = reinterpret_cast<const uint16_t*>(P.proj[U.p].blob + U.w16_off);
                for (int m = warp; m < U.n16; m += kT1Warps)
                    acc = fmaf(s_c16[m], __half2float(__ushort_as_half(w16[(size_t)m * P.d_pad + row])), acc);
            }
        }
        s_part[warp * kRB + lane] = acc;
        __syncthreads();
        if (warp == 0) {
            float y = 0.0f;
            if (U.e >= 0) {
#pragma unroll
                for (int w = 0; w < kT1Warps; w++) y += s_part[w * kRB + lane];
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
    P.tasks_max = (P.n_tasks + P.G - 1) / P.G;
    int pw = 0, members = 0, meta = 0, n16 = 0;
    unit_bounds(g, pw, members, meta, n16);
    unit_bounds(u, pw, members, meta, n16);
    P.pw_max = pw;
    P.members_max = members;
    P.meta_max = align_up(meta, 16);
    P.n16_max = n16;
    const int units_max = (P.tasks_max + P.n_rb - 1) / P.n_rb + 1;
    if (units_max > kMaxUnitsPerCta || P.tasks_max > 64 || P.d_in % 8 || P.d_in > 8192) return L;
    // shared memory
    const uint64_t phi_bytes = (uint64_t)P.phi_rows * P.d_in * 2;
    P.a_z = 0;
    P.a_tab = align_up(P.a_z + 8ull * P.r, 128);
    P.a_part = align_up(P.a_tab + 64 + 16ull * 4 * (members / 4), 16);  // + 64: tables realigned in the kernel
    P.a_c16 = align_up(P.a_part + 4ull * kT1Warps * kRB, 16);
    P.a_desc = align_up(P.a_c16 + 4ull * n16, 16);
    const uint64_t a_bytes = std::max<uint64_t>(phi_bytes, P.a_desc + 8ull * P.pw_max);
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
