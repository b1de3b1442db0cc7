// layer_t1.cu -- fused single-token layer forward: both projections, one
// persistent launch (one CTA per SM).
//
// The method (BitsMoE study-note page, Methodology, first split; second
// split; Execution): z = Phi^T x is computed once per token and reused by the
// token's top-k experts; each expert evaluates its width-grouped bit planes
// bit-serially:  y_i = sum_b sum_j 2^j sum_{k in G_b} c_k bit_{k,j,i}
//                      - sum_b (2^b - 1)/2 sum_{k in G_b} c_k,  c_k = a_k s_k z_k.
//
// Design for B200 at one token.  The step moves ~24 MB (Phi of both
// projections dominates) and one grid-wide dependency (expert rows need z
// rows that other CTAs compute).  Every CTA issues its HBM reads at launch --
// its slice of Phi rows, its share of the routed bit planes and their
// metadata, all by bulk copies -- and computes its z rows.  There is no grid
// barrier: each z row is published as one 64-bit word carrying the launch's
// tag next to the value, and a CTA polls exactly the z words its members need,
// so the wait and the gather are one L2 round trip.
//
// The expert work is cut by COLUMNS: the routed units' plane words (one word
// = one bit plane of 32 members, over all rows) and octets of fp16 members
// are concatenated and every CTA takes an equal contiguous share of them, for
// all rows.  So a CTA builds subset-sum tables only for the member words it
// evaluates (no table is built twice except at share boundaries), and the
// work per CTA differs by at most one word.  Warps own 32-row tiles; the sum
// over 32 members of one plane word uses eight 16-entry tables (one per
// nibble), one shared-memory lookup per 4 bits.  Each CTA adds its rows of
// every unit it touched (with its share of the zero-point term subtracted) to
// Y_e and, times the gate weight, to Y_sum with fp32 red.add, after acquiring
// the tags the CTAs that zeroed the outputs published; the order of those
// additions, and so the last bits of the outputs, can differ from run to run.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"

namespace bitsmoe {

constexpr int kT1MaxThreads = 768;
constexpr int kT1MaxWarps = kT1MaxThreads / 32;
constexpr int kRB = 32;           // rows per tile (one per lane)
constexpr int kMaxUnits = 32;     // routed (projection, slot) pairs: 2 * top_k
constexpr int kMaxItems = 32;     // work items per CTA (one planning lane each)
constexpr int kF16Item = 8;       // fp16 members per item
constexpr int kStageWarps = 1;    // warps that issue the plane and metadata copies
constexpr int kPhiBars = 4;       // mbarriers over the Phi slice
constexpr long long kWaitLimitNs = 2000000000LL;  // bounded waits: 2 s, then BITSMOE_ST_TIMEOUT
constexpr int kTagBar = kPhiBars + 3;  // mbarrier that hands this launch's tag to the row warps
constexpr int kMaxZeroCtas = 16;       // CTAs that zero the outputs (each publishes a tag)
constexpr int kZeroSliceFloats = 16384;  // outputs zeroed per zeroing CTA, at least
// workspace head: [0] launch counter, [1 .. kMaxZeroCtas] the zeroing CTAs' tags
static_assert(8 * (1 + kMaxZeroCtas) <= 256, "the workspace head is 256 bytes");

struct T1Proj {
    const uint8_t* blob;
    const uint16_t* phi_t;
    float* Z;     // [r] or null
    float* Ye;    // [K][d_out] or null
    float* Ysum;  // [d_out]
};

struct T1Params {
    T1Proj proj[2];
    const uint16_t* next_phi[2];  // the next layer's Phi^T (both projections) to prefetch into L2, or null
    const uint16_t* x;
    const int32_t* ids;
    const float* gw;
    int32_t* status;
    unsigned long long* launches;   // persistent, zero-initialised once; every CTA adds 1 per launch
    unsigned long long* zero_tags;  // [n_zero]: tag of the last launch whose outputs each zeroing CTA cleared
    unsigned long long* zbuf;       // [2][r] z rows, each (launch tag << 32) | fp32 bits
    int d_in, d_out, d_pad, r, K, E, U;
    int n_rb, G;
    int n_zero;     // CTAs that zero the outputs (1 .. kMaxZeroCtas)
    int items_max;  // work items per CTA (upper bound over every routing)
    // dynamic shared-memory layout (byte offsets)
    uint32_t sm_x, sm_dir, sm_phi, sm_planes, sm_mw, sm_f16, sm_c16, sm_tab, sm_end;
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
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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
// Bulk copy global -> shared with an L2 cache policy (createpolicy).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}
// Streamed data (Phi, bit planes) is read once per step: evict it first.  The
// expert directories are tiny and read by every CTA of every step: keep them.
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// Named barrier `ID` over n threads (whole warps).  The callers come out of code
// whose trip counts differ between lanes, so the warp is reconverged first:
// bar.sync wants all 32 lanes to execute it together.
template <int ID>
__device__ __forceinline__ void named_barrier(int n) {
    __syncwarp();
    asm volatile("bar.sync %0, %1;" ::"n"(ID), "r"(n) : "memory");
}
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void red_add_f32(float* p, float v) {
    asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}
// Shared load at a 32-bit shared address plus a constant byte offset.  Not
// volatile, so the compiler may schedule it; its address always derives from a
// descriptor read after the barrier that publishes the tables.
template <int OFF>
__device__ __forceinline__ float lds_f32_imm(uint32_t addr) {
    float v;
    asm("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(OFF));
    return v;
}
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
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// Bounded spin until *p holds tag (acquire); false on timeout.
__device__ __forceinline__ bool tag_wait(const unsigned long long* p, unsigned long long tag) {
    if (ld_acquire_u64(p) == tag) return true;
    const long long t0 = globaltimer();
    while (ld_acquire_u64(p) != tag)
        if (globaltimer() - t0 > kWaitLimitNs) return false;
    return true;
}
// z row k of this launch: a z word is one 64-bit store of (tag << 32) | value,
// so the load that sees this launch's tag also sees its value.  Polls (bounded;
// on timeout, or once another thread of the CTA timed out, sets *timed_out and
// returns 0).
__device__ __forceinline__ float z_poll(const unsigned long long* w, uint32_t tag, volatile int* timed_out) {
    unsigned long long v = ld_relaxed_u64(w);
    if ((uint32_t)(v >> 32) != tag) {
        const long long t0 = globaltimer();
        while ((uint32_t)((v = ld_relaxed_u64(w)) >> 32) != tag) {
            if (*timed_out || globaltimer() - t0 > kWaitLimitNs) {
                *timed_out = 1;
                return 0.0f;
            }
        }
    }
    return __uint_as_float((uint32_t)v);
}

// ---------------------------------------------------------------------------
// routed units and the column partition
// ---------------------------------------------------------------------------
// One routed (projection, slot) pair.
struct UnitInfo {
    int p, j, e;  // projection, slot, expert (-1 when the id is out of range)
    float g;      // gate weight
    int pw;       // plane words
    int n16;      // fp16 members
    int items;    // plane words + octets of fp16 members
    uint32_t np[kNumGroups], n[kNumGroups], pw0[kNumGroups];
    uint64_t gbase[kNumGroups];  // byte offset of each group in the blob
};

__device__ inline void unit_info(const T1Params& P, int u, int e, const uint8_t* s_dir, UnitInfo& U) {
    U.p = u / P.K;
    U.j = u % P.K;
    U.e = (e >= 0 && e < P.E) ? e : -1;
    U.g = P.gw[U.j];
    U.pw = U.n16 = U.items = 0;
    for (int g = 0; g < kNumGroups; g++) {
        U.np[g] = U.n[g] = U.pw0[g] = 0;
        U.gbase[g] = 0;
    }
    if (U.e < 0) return;
    const DirEntry d = parse_dir(s_dir + ((size_t)U.p * P.E + U.e) * kDirEntryBytes);
    uint32_t pw = 0;
    for (int g = 0; g < kNumGroups; g++) {
        const int b = group_width(g);
        U.n[g] = d.count[g];
        U.np[g] = (uint32_t)group_members_padded(b, d.count[g]);
        U.pw0[g] = pw;
        U.gbase[g] = d.base + d.goff[g];
        if (b != 16) pw += (uint32_t)b * (U.np[g] / 32);
    }
    U.pw = (int)pw;
    U.n16 = (int)U.n[0];
    U.items = U.pw + (U.n16 + kF16Item - 1) / kF16Item;
}

// Plane word q of a unit -> (group, bit plane, word).  Words are ordered by
// group, then plane, then word.
__device__ __forceinline__ void decode_pw(const UnitInfo& U, int q, int& g, int& jb, int& w) {
    g = 1;
#pragma unroll
    for (int gg = 2; gg < kNumGroups; gg++)
        if ((uint32_t)q >= U.pw0[gg] && U.np[gg] > 0) g = gg;
    const int W = (int)(U.np[g] / 32);
    const int rel = q - (int)U.pw0[g];
    jb = rel / W;
    w = rel - jb * W;
}

// One work item of a CTA: a plane word (all rows of one bit plane of 32
// members) or an octet of fp16 members (all rows).
struct Item {
    const uint8_t* ptr;  // plane word: its d_pad words (one per row); octet: member row 8f
    int16_t nf;          // octet: fp16 members in it (1..8); plane word: 0
    int16_t slot;        // member-word slot (plane word) or octet slot
    int16_t w;           // octet: f
    int16_t u;           // unit
};
// A member word (32 members of a group) whose c values and tables this CTA builds.
struct MemberWord {
    int16_t p, g, w;
    int16_t nvalid;  // real members in the word (0..32)
    int16_t zp;      // 1 when this CTA evaluates the word's plane 0 and so owns its zero-point share
    int16_t seg;
};
// Consecutive plane-word items of one group: contiguous in the blob (planes
// are [b][W][d_pad], rows fastest), so one bulk copy stages all of them.
struct Run {
    const uint8_t* ptr;  // the first item's words
    int a, len;          // first item slot, items
};
// Consecutive member-word slots of one group with consecutive words: their idx,
// scale and amp are each one contiguous block in the blob and in shared memory.
struct MetaRun {
    const uint8_t* meta;  // the group's metadata
    uint32_t np;          // padded members of the group
    int w, slot, len;     // first word, first slot, words
};
// Items of one unit inside a CTA's share: plane words [i0, ip), fp16 octets [ip, i1).
struct Seg {
    int u, i0, ip, i1;
};

// acc0 += the products of the low halves of the four fp16 pairs of a and b,
// acc1 += those of the high halves: mixed-precision FMAs (fp16 operands, exact
// in fp32; fp32 addend), so no fp16 value is converted on its own.
__device__ __forceinline__ void dot8_f16(const uint4 a, const uint4 b, float& acc0, float& acc1) {
    asm("{\n"
        " .reg .f16 a0, a1, a2, a3, a4, a5, a6, a7, b0, b1, b2, b3, b4, b5, b6, b7;\n"
        " mov.b32 {a0, a1}, %2;\n mov.b32 {a2, a3}, %3;\n mov.b32 {a4, a5}, %4;\n mov.b32 {a6, a7}, %5;\n"
        " mov.b32 {b0, b1}, %6;\n mov.b32 {b2, b3}, %7;\n mov.b32 {b4, b5}, %8;\n mov.b32 {b6, b7}, %9;\n"
        " fma.rn.f32.f16 %0, a0, b0, %0;\n fma.rn.f32.f16 %1, a1, b1, %1;\n"
        " fma.rn.f32.f16 %0, a2, b2, %0;\n fma.rn.f32.f16 %1, a3, b3, %1;\n"
        " fma.rn.f32.f16 %0, a4, b4, %0;\n fma.rn.f32.f16 %1, a5, b5, %1;\n"
        " fma.rn.f32.f16 %0, a6, b6, %0;\n fma.rn.f32.f16 %1, a7, b7, %1;\n"
        "}"
        : "+f"(acc0), "+f"(acc1)
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w));
}

// Items [q0, q1) of CTA c out of Q: an equal contiguous share.  c * Q stays
// below 2^32 for every shape the fused path takes (the host checks it).
__host__ __device__ __forceinline__ int share_begin(int c, int Q, int G) {
    return (int)(((uint32_t)c * (uint32_t)Q) / (uint32_t)G);
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kT1MaxThreads, 1) k_layer_t1(const T1Params P) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t s_bar[kPhiBars + 4];  // Phi chunks, the expert directories, planes, metadata, tag
    __shared__ Run s_run[kMaxItems];
    __shared__ MetaRun s_mrun[kMaxItems];
    __shared__ UnitInfo s_unit[kMaxUnits];
    __shared__ Item s_item[kMaxItems];
    __shared__ MemberWord s_mw[kMaxItems];
    __shared__ Seg s_seg[kMaxItems];
    __shared__ uint2 s_desc[kMaxItems];  // plane word: (tables' shared address, 2^j bits)
    __shared__ float s_zpmw[kMaxItems];
    __shared__ int s_ni, s_nmw, s_nseg, s_nrun, s_nmrun, s_abort, s_bad;
    __shared__ volatile int s_zto;  // a z poll timed out
    __shared__ uint32_t s_stage_bytes, s_meta_bytes;
    __shared__ uint32_t s_tag;      // this launch's tag (1 .. 2^32 - 1)

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nthreads = blockDim.x, nwarps = nthreads >> 5;
    const int cta = blockIdx.x;
    const int row0 = share_begin(cta, 2 * P.r, P.G), row1 = share_begin(cta + 1, 2 * P.r, P.G);
    const int nrows = row1 - row0;
    const uint32_t row_bytes = (uint32_t)P.d_in * 2;

    uint16_t* s_x = reinterpret_cast<uint16_t*>(smem + P.sm_x);
    uint8_t* s_dir = smem + P.sm_dir;  // [projection][expert] directory entries
    uint8_t* s_phi = smem + P.sm_phi;
    uint32_t* s_planes = reinterpret_cast<uint32_t*>(smem + P.sm_planes);  // [item slot][d_pad]
    // member-word metadata, one array each, 32 members per slot
    uint16_t* s_midx = reinterpret_cast<uint16_t*>(smem + P.sm_mw);
    uint16_t* s_mscl = s_midx + 32 * P.items_max;
    float* s_mamp = reinterpret_cast<float*>(s_mscl + 32 * P.items_max);
    uint8_t* s_f16d = smem + P.sm_f16;  // [octet]: idx u16[8] | amp f32[8]
    float* s_c16 = reinterpret_cast<float*>(smem + P.sm_c16);  // [octet][8]
    // tables start on a 512-byte shared-memory boundary: one member word's 8
    // tables are 512 B, so the byte address of a word's tables has a zero low
    // byte and a lookup can splice the entry offset into it with one byte permute
    uint8_t* tab_raw = smem + P.sm_tab;
    float* s_tab = reinterpret_cast<float*>(tab_raw + ((512u - (smem_u32(tab_raw) & 511u)) & 511u));
    const uint32_t tab_sbase = smem_u32(s_tab);

    // ---- phase 0: the routed ids are loaded first; one thread initialises the
    // mbarriers and then issues the Phi rows and x (they need nothing) ----
    const int my_id = (warp == 1 && lane < P.U) ? P.ids[lane % P.K] : 0;
    if (tid == 0) {
        for (int i = 0; i < kPhiBars + 4; i++) mbar_init(&s_bar[i], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_abort = 0;
        s_zto = 0;
    }
    __syncthreads();  // the mbarriers are initialised
    // Roles: warp 1 plans this CTA's share and hands it to the last kStageWarps
    // warps, which issue the staging copies; the other warps compute z rows as
    // the Phi chunks land.  The three run side by side.
    const int nrw = nwarps - kStageWarps;  // warps before the staging warps
    const bool row_warp = warp < nrw;
    if (tid == 0) {
        // both expert directories first: the routed units need them before anything else
        const uint32_t dir_bytes = (uint32_t)P.E * kDirEntryBytes;
        const uint64_t keep = policy_evict_last(), stream = policy_evict_first();
        mbar_expect_tx(&s_bar[kPhiBars], 2 * dir_bytes);
        for (int p = 0; p < 2; p++)
            bulk_g2s(s_dir + (size_t)p * dir_bytes, P.proj[p].blob + kHeaderBytes, dir_bytes, &s_bar[kPhiBars], keep);
        for (int bi = 0; bi < kPhiBars; bi++) {
            const int ra = row0 + (nrows * bi) / kPhiBars, rbnd = row0 + (nrows * (bi + 1)) / kPhiBars;
            const uint32_t bytes = (uint32_t)(rbnd - ra) * row_bytes + (bi == 0 ? row_bytes : 0);
            mbar_expect_tx(&s_bar[bi], bytes);
            if (bi == 0) bulk_g2s(s_x, P.x, row_bytes, &s_bar[0], stream);
            for (int rr = ra; rr < rbnd;) {  // rows are contiguous inside a projection
                const int p = rr / P.r, k = rr - p * P.r;
                const int n = min(rbnd - rr, P.r - k);
                bulk_g2s(s_phi + (size_t)(rr - row0) * row_bytes, P.proj[p].phi_t + (size_t)k * P.d_in,
                         (uint32_t)n * row_bytes, &s_bar[bi], stream);
                rr += n;
            }
        }
        // This launch's tag.  Every launch adds exactly G to the counter (one per
        // CTA, whatever happens later), so before this CTA's addition it holds G
        // times the number of earlier launches n plus fewer than G of this one's.
        // The tag, n mod (2^32 - 1) plus 1, is never 0 (a zero-filled z word) and
        // never that of the launch before.
        const unsigned long long before = atomicAdd(P.launches, 1ull);
        s_tag = (uint32_t)((before / (unsigned long long)P.G) % 0xFFFFFFFFull) + 1u;
        mbar_arrive(&s_bar[kTagBar]);  // publishes s_tag to the row warps
    }

    // ---- routed units and this CTA's share (warp 1; one lane per unit, then per item).
    // The other warps wait: this is short, and alone on the SM it is not slowed by them ----
    if (warp == 1) {
        const bool dir_ok = mbar_wait(&s_bar[kPhiBars], 0);
        if (lane < P.U) unit_info(P, lane, dir_ok ? my_id : -1, s_dir, s_unit[lane]);
        if (!dir_ok && lane == 0) s_abort = 1;
        __syncwarp();
        const bool is_unit = lane < P.U;
        const int my_items = is_unit ? s_unit[lane].items : 0;
        int incl = my_items;  // inclusive scan of items over units
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int excl = incl - my_items;
        const int Q = __shfl_sync(0xffffffffu, incl, 31);
        const int q0 = share_begin(cta, Q, P.G);
        int ni = share_begin(cta + 1, Q, P.G) - q0;
        if (ni > P.items_max || ni > kMaxItems) {  // the blob's counts disagree with the plan's
            if (lane == 0 && P.status) atomicOr(P.status, BITSMOE_ST_PLANMISMATCH);
            ni = 0;
        }
        const bool bad = __any_sync(0xffffffffu, is_unit && s_unit[lane].e < 0);
        // unit of item `lane`: the number of units that end at or before it
        int my_u = 0;
#pragma unroll
        for (int v = 0; v < 32; v++) my_u += (v < P.U && __shfl_sync(0xffffffffu, incl, v) <= q0 + lane) ? 1 : 0;
        my_u = min(my_u, P.U - 1);
        const int S_u = __shfl_sync(0xffffffffu, excl, my_u & 31);
        const bool valid = lane < ni;
        Item it{};
        int key = -1 - lane, g = 0, jb = -1, w = 0;  // member-word key of a plane word; unique otherwise
        if (valid) {
            const UnitInfo& U = s_unit[my_u];
            const int l = q0 + lane - S_u;
            const uint8_t* blob = P.proj[U.p].blob;
            it.u = (int16_t)my_u;
            if (l < U.pw) {
                decode_pw(U, l, g, jb, w);
                const uint32_t W = U.np[g] / 32;
                it.ptr = blob + U.gbase[g] + 8ull * U.np[g] + 4ull * P.d_pad * ((uint64_t)jb * W + (uint64_t)w);
                it.nf = 0;
                key = (my_u << 24) | (g << 16) | w;
            } else {
                const int f = l - U.pw;
                it.ptr = blob + U.gbase[0] + 6ull * U.np[0] + 2ull * kF16Item * (uint64_t)f * (uint64_t)P.d_pad;
                it.nf = (int16_t)min(kF16Item, U.n16 - kF16Item * f);
                it.w = (int16_t)f;
            }
        }
        const bool plane = valid && it.nf == 0, oct = valid && it.nf > 0;
        // runs of plane words: consecutive items whose words follow each other in the blob
        const uint64_t my_ptr = (uint64_t)it.ptr;
        const uint64_t prev_ptr = __shfl_up_sync(0xffffffffu, my_ptr, 1);
        const int prev_plane = __shfl_up_sync(0xffffffffu, (int)plane, 1);
        const bool cont = plane && lane > 0 && prev_plane && my_ptr == prev_ptr + 4ull * P.d_pad;
        const unsigned bcont = __ballot_sync(0xffffffffu, cont), bplane = __ballot_sync(0xffffffffu, plane);
        const unsigned brun = bplane & ~bcont;
        if ((brun >> lane) & 1u) {
            const unsigned stop = ~bcont & (lane == 31 ? 0u : ~((2u << lane) - 1u));  // first later item not continuing
            Run R;
            R.ptr = it.ptr;
            R.a = lane;
            R.len = (stop ? __ffs(stop) - 1 : 32) - lane;
            s_run[__popc(brun & ((1u << lane) - 1u))] = R;
        }
        if (lane == 0) {
            s_nrun = __popc(brun);
            s_stage_bytes = 4u * (uint32_t)P.d_pad * (uint32_t)__popc(bplane);
        }
        named_barrier<2>(32 * (1 + kStageWarps));  // the plane runs are known: the staging warps copy them now
        // first item of the same member word, and whether any of them is plane 0
        int ref = lane, zp = 0;
        const int z0 = plane && jb == 0;
#pragma unroll
        for (int k = 0; k < 32; k++) {
            const int kk = __shfl_sync(0xffffffffu, key, k), kz = __shfl_sync(0xffffffffu, z0, k);
            if (k < ni && kk == key) {
                if (k < ref) ref = k;
                zp |= kz;
            }
        }
        const unsigned lt = (1u << lane) - 1u;
        const bool newmw = plane && ref == lane;
        const unsigned bm = __ballot_sync(0xffffffffu, newmw), bf = __ballot_sync(0xffffffffu, oct);
        const int slot_new = __popc(bm & lt);
        const int slot_ref = __shfl_sync(0xffffffffu, slot_new, ref);
        const int slot = oct ? __popc(bf & lt) : slot_ref;
        const int u_prev = __shfl_up_sync(0xffffffffu, my_u, 1);
        const bool newseg = valid && (lane == 0 || u_prev != my_u);
        const unsigned bs = __ballot_sync(0xffffffffu, newseg);
        const int seg = __popc(bs & (lt | (1u << lane))) - 1;
        if (valid) {
            it.slot = (int16_t)slot;
            s_item[lane] = it;
            s_desc[lane] = plane ? make_uint2(tab_sbase + 512u * (uint32_t)slot, __float_as_uint((float)(1u << jb)))
                                 : make_uint2(0u, 0u);
        }
        if (newmw) {
            const UnitInfo& U = s_unit[my_u];
            MemberWord M;
            M.p = (int16_t)U.p;
            M.g = (int16_t)g;
            M.w = (int16_t)w;
            M.nvalid = (int16_t)max(0, min(32, (int)U.n[g] - 32 * w));
            M.zp = (int16_t)zp;
            M.seg = (int16_t)seg;
            s_mw[slot_new] = M;
        }
        {   // runs of member words in slot order: consecutive slots, same group, consecutive words
            const unsigned below = bm & lt;
            const int prev = below ? 31 - __clz(below) : 0;  // the previous slot's lane
            const int pkey = __shfl_sync(0xffffffffu, key, prev);
            const bool mcont = newmw && below != 0u && pkey == key - 1;
            const unsigned bmc = __ballot_sync(0xffffffffu, mcont);
            const unsigned bmr = bm & ~bmc;  // run starts
            if ((bmr >> lane) & 1u) {
                const unsigned after = lane == 31 ? 0u : ~((2u << lane) - 1u);
                const unsigned nxt = bmr & after;
                const unsigned span = nxt ? (after & ((1u << (__ffs(nxt) - 1)) - 1u)) : after;
                const UnitInfo& U = s_unit[my_u];
                MetaRun R;
                R.meta = P.proj[U.p].blob + U.gbase[g];
                R.np = U.np[g];
                R.w = w;
                R.slot = slot_new;
                R.len = 1 + __popc(bm & span);
                s_mrun[__popc(bmr & lt)] = R;
            }
            if (lane == 0) s_nmrun = __popc(bmr);
        }
        if (newseg) {
            const unsigned above = bs & ~(lt | (1u << lane));
            const int i1 = above ? __ffs(above) - 1 : ni;
            const unsigned in_seg = (i1 >= 32 ? 0xffffffffu : ((1u << i1) - 1u)) & ~lt;
            const unsigned octs = bf & in_seg;
            Seg S;
            S.u = my_u;
            S.i0 = lane;
            S.i1 = i1;
            S.ip = octs ? __ffs(octs) - 1 : i1;
            s_seg[seg] = S;
        }
        if (lane == 0) {
            s_ni = ni;
            s_nmw = __popc(bm);
            s_nseg = __popc(bs);
            s_meta_bytes = 256u * __popc(bm) + 48u * __popc(bf);
            s_bad = bad;
        }
        named_barrier<3>(32 * (1 + kStageWarps));  // the rest of the plan: member words and octets
    }

    // ---- the outputs are sums of red.add contributions: the first n_zero CTAs zero
    // them and then publish this launch's tag; every CTA acquires those tags before
    // its first addition ----
    const int rw = warp == 0 ? 0 : warp - 1, nrw1 = nrw - 1;  // index and count of the z-row warps
    if (cta < P.n_zero && row_warp && warp != 1) {
        const int nys = 2 * P.d_out;
        const int nye0 = P.proj[0].Ye ? P.K * P.d_out : 0, nye1 = P.proj[1].Ye ? P.K * P.d_out : 0;
        const int tot = nys + nye0 + nye1;
        const int a = share_begin(cta, tot, P.n_zero), b = share_begin(cta + 1, tot, P.n_zero);
        for (int i = a + rw * 32 + lane; i < b; i += nrw1 * 32) {
            float* dst;
            if (i < P.d_out)
                dst = P.proj[0].Ysum + i;
            else if (i < nys)
                dst = P.proj[1].Ysum + (i - P.d_out);
            else if (i < nys + nye0)
                dst = P.proj[0].Ye + (i - nys);
            else
                dst = P.proj[1].Ye + (i - nys - nye0);
            *dst = 0.0f;
        }
        // the row warps' zeros are ordered before the tag by this CTA barrier and
        // the cumulative release of the store (thread 0 wrote s_tag itself)
        named_barrier<4>(nrw1 * 32);
        if (tid == 0) st_release_u64(P.zero_tags + cta, (unsigned long long)s_tag);
    }

    // ---- staging by the staging warp (bulk copies on one mbarrier): each run of plane
    // words in one copy into [item slot][d_pad]; each run of member words' idx, scale
    // and amp in one copy per array; each octet's idx and amp ----
    if (!row_warp) {
        named_barrier<2>(32 * (1 + kStageWarps));
        // A CTA's bulk copies land in about the order they are issued, so copies
        // issued now would land after this CTA's Phi rows anyway; issued now they
        // would also take HBM time from other CTAs' Phi rows, which every CTA
        // waits for.  So they are issued once this CTA's last Phi chunk has landed.
        const bool phi_ok = mbar_wait(&s_bar[kPhiBars - 1], 0);
        if (!phi_ok) s_abort = 1;
        const int st = threadIdx.x - nrw * 32, nst = kStageWarps * 32;
        const uint64_t stream = policy_evict_first();
        uint64_t* bar = &s_bar[kPhiBars + 1];
        if (st == 0) mbar_expect_tx(bar, s_stage_bytes);
        __syncwarp();
        for (int r = st; r < s_nrun; r += nst) {
            const Run R = s_run[r];
            bulk_g2s(s_planes + (size_t)R.a * P.d_pad, R.ptr, 4u * (uint32_t)P.d_pad * (uint32_t)R.len, bar, stream);
        }
        named_barrier<3>(32 * (1 + kStageWarps));
        const int ni = s_ni;
        bar = &s_bar[kPhiBars + 2];
        if (st == 0) mbar_expect_tx(bar, s_meta_bytes);
        __syncwarp();
        for (int r = st; r < s_nmrun; r += nst) {
            const MetaRun R = s_mrun[r];
            const uint32_t n = (uint32_t)R.len;
            bulk_g2s(s_midx + 32 * R.slot, R.meta + 64ull * R.w, 64u * n, bar, stream);                // idx
            bulk_g2s(s_mscl + 32 * R.slot, R.meta + 2ull * R.np + 64ull * R.w, 64u * n, bar, stream);  // scale
            bulk_g2s(s_mamp + 32 * R.slot, R.meta + 4ull * R.np + 128ull * R.w, 128u * n, bar, stream);  // amp
        }
        for (int i = st; i < ni; i += nst) {
            const Item& it = s_item[i];
            if (!it.nf) continue;
            const UnitInfo& U = s_unit[it.u];
            const uint8_t* gb = P.proj[U.p].blob + U.gbase[0];
            uint8_t* dst = s_f16d + 48 * it.slot;
            bulk_g2s(dst, gb + 16ull * it.w, 16u, bar, stream);
            bulk_g2s(dst + 16, gb + 2ull * U.np[0] + 32ull * it.w, 32u, bar, stream);
        }
    }

    // ---- phase 1: z rows of this CTA (row warps), each published with this launch's tag ----
    if (row_warp && warp != 1) {
        bool ok = nrows == 0 || (mbar_wait(&s_bar[kTagBar], 0) && mbar_wait(&s_bar[0], 0));  // 0 carries x
        const unsigned long long tag_hi = (unsigned long long)s_tag << 32;
        for (int rl = rw; ok && rl < nrows; rl += nrw1) {
            int bi = 0;
            while (bi + 1 < kPhiBars && rl >= (nrows * (bi + 1)) / kPhiBars) bi++;
            if (!mbar_wait(&s_bar[bi], 0)) {
                ok = false;
                break;
            }
            const uint4* rowv = reinterpret_cast<const uint4*>(s_phi + (size_t)rl * row_bytes);
            const uint4* xv = reinterpret_cast<const uint4*>(s_x);
            float acc = 0.0f, acc1 = 0.0f;
            for (int i8 = lane; i8 < P.d_in / 8; i8 += 32) dot8_f16(rowv[i8], xv[i8], acc, acc1);
            acc = warp_sum(acc + acc1);
            if (lane == 0) {
                const int rr = row0 + rl, p = rr / P.r, k = rr - p * P.r;
                st_relaxed_u64(P.zbuf + rr, tag_hi | __float_as_uint(acc));
                if (P.proj[p].Z) P.proj[p].Z[k] = acc;
            }
        }
        if (!ok) s_abort = 1;
        named_barrier<1>(nrw1 * 32);
        if (tid == 0)
            for (int bi = 0; bi < kPhiBars; bi++)  // every bulk copy into this CTA's shared memory has landed
                if (!mbar_wait(&s_bar[bi], 0)) s_abort = 1;
    }
    __syncthreads();
    const int ni = s_ni, nmw = s_nmw, nseg = s_nseg;
    const uint32_t tag = s_tag;

    // ---- the outputs are zeroed, the planes and metadata have landed (bounded waits) ----
    if (tid == 0) {
        for (int z = 0; z < P.n_zero; z++)
            if (!tag_wait(P.zero_tags + z, (unsigned long long)tag)) s_abort = 1;
        if (!mbar_wait(&s_bar[kPhiBars + 1], 0)) s_abort = 1;  // the staged planes
        if (!mbar_wait(&s_bar[kPhiBars + 2], 0)) s_abort = 1;  // and metadata
        if (s_bad && cta == 0 && P.status) atomicOr(P.status, BITSMOE_ST_BADEXPERT);
    }
    __syncthreads();
    if (s_abort) {
        if (tid == 0 && P.status) atomicOr(P.status, BITSMOE_ST_TIMEOUT);
        return;
    }

    // ---- c_k = a_k s_k z_k, the tables and the zero-point share: a warp per member word ----
    for (int m = warp; m < nmw; m += nwarps) {
        const MemberWord M = s_mw[m];
        const int k = s_midx[32 * m + lane];
        float c = 0.0f;
        if (lane < M.nvalid && k < P.r)
            c = s_mamp[32 * m + lane] * __half2float(__ushort_as_half(s_mscl[32 * m + lane])) *
                z_poll(P.zbuf + M.p * P.r + k, tag, &s_zto);
        // entry e of table tb = the sum of c over the set bits of e (members 4 tb .. 4 tb + 3)
        const int e = lane & 15;
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const int tb = (lane >> 4) + 2 * q;
            const float c0 = __shfl_sync(0xffffffffu, c, 4 * tb), c1 = __shfl_sync(0xffffffffu, c, 4 * tb + 1);
            const float c2 = __shfl_sync(0xffffffffu, c, 4 * tb + 2), c3 = __shfl_sync(0xffffffffu, c, 4 * tb + 3);
            s_tab[128 * m + 16 * tb + e] =
                ((e & 1 ? c0 : 0.0f) + (e & 2 ? c1 : 0.0f)) + ((e & 4 ? c2 : 0.0f) + (e & 8 ? c3 : 0.0f));
        }
        float h = M.zp ? 0.5f * (float)((1 << group_width(M.g)) - 1) * c : 0.0f;
        h = warp_sum(h);
        if (lane == 0) s_zpmw[m] = h;
    }
    for (int ch = tid; ch < ni * kF16Item; ch += nthreads) {
        const int i = ch / kF16Item, m = ch - i * kF16Item;
        const Item& it = s_item[i];
        if (!it.nf) continue;
        const uint8_t* fd = s_f16d + 48 * it.slot;
        const int k = reinterpret_cast<const uint16_t*>(fd)[m];
        float c = 0.0f;
        if (m < it.nf && k < P.r)
            c = reinterpret_cast<const float*>(fd + 16)[m] * z_poll(P.zbuf + s_unit[it.u].p * P.r + k, tag, &s_zto);
        s_c16[kF16Item * it.slot + m] = c;
    }
    __syncthreads();
    if (s_zto) {
        if (tid == 0 && P.status) atomicOr(P.status, BITSMOE_ST_TIMEOUT);
        return;
    }
    // This CTA has every z row it needs, so the Phi reads of this launch are all
    // but done: HBM is free while the experts are evaluated, so pull this CTA's
    // rows of the next layer's Phi into L2 for the next call.
    if (tid == 0 && P.next_phi[0] && P.next_phi[1])
        for (int rr = row0; rr < row1;) {
            const int p = rr / P.r, k = rr - p * P.r;
            const int n = min(row1 - rr, P.r - k);
            bulk_prefetch_l2(P.next_phi[p] + (size_t)k * P.d_in, (uint32_t)n * row_bytes);
            rr += n;
        }

    // ---- lookups: warps own 32-row tiles; a segment's rows go to Y_e and, times g, to Y_sum ----
    for (int s = 0; s < nseg; s++) {
        const Seg S = s_seg[s];
        const UnitInfo& U = s_unit[S.u];
        const int p = U.p;
        float* ye = P.proj[p].Ye ? P.proj[p].Ye + (size_t)U.j * P.d_out : nullptr;
        float* ys = P.proj[p].Ysum;
        const float gj = U.g;
        // this CTA's zero-point share of the unit (member words in slot order)
        const float zps = warp_sum(lane < nmw && s_mw[lane].seg == s ? s_zpmw[lane] : 0.0f);
        for (int t = warp; t < P.n_rb; t += nwarps) {
            const uint32_t* pl = s_planes + t * kRB + lane;  // [item slot][d_pad]
            float acc = 0.0f;
#pragma unroll 4
            for (int i = S.i0; i < S.ip; i++) {
                const uint2 d = s_desc[i];
                const uint32_t word = pl[i * P.d_pad];
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
                acc = fmaf(sum, __uint_as_float(d.y), acc);
            }
            const int row = t * kRB + lane;
            for (int i = S.ip; i < S.i1; i++) {  // fp16 octets, rows read in place
                const Item& it = s_item[i];
                const uint16_t* w16 = reinterpret_cast<const uint16_t*>(it.ptr);
                for (int m = 0; m < it.nf; m++)
                    acc = fmaf(s_c16[kF16Item * it.slot + m],
                               __half2float(__ushort_as_half(w16[(size_t)m * P.d_pad + row])), acc);
            }
            if (row < P.d_out) {
                const float y = acc - zps;
                if (ye) red_add_f32(ye + row, y);
                red_add_f32(ys + row, gj * y);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct T1Layout {
    bool ok;
    T1Params P;
    uint64_t ws_reserved;  // persistent counter at the start of the workspace
    size_t smem;
    int threads;
};

static int g_num_sms = 0;
static int g_max_smem = 0;
static int g_static_smem = -1;

// Largest dynamic shared memory size k_layer_t1 has been granted on each
// device, so that a launch asks the runtime again only when it needs more.
constexpr int kMaxDevices = 256;
static std::atomic<int> g_smem_granted[kMaxDevices];

static cudaError_t grant_smem(int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool cached = dev >= 0 && dev < kMaxDevices;
    if (cached && g_smem_granted[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(k_layer_t1, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess || !cached) return e;
    int prev = g_smem_granted[dev].load(std::memory_order_relaxed);
    while (prev < bytes && !g_smem_granted[dev].compare_exchange_weak(prev, bytes)) {
    }
    return cudaSuccess;
}

static bool device_info() {
    if (g_num_sms > 0 && g_static_smem >= 0) return true;
    int dev;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&g_max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, k_layer_t1) != cudaSuccess) return false;
    g_static_smem = (int)fa.sharedSizeBytes;
    return true;
}

// Work items (plane words + fp16 octets) of the largest expert of a plan,
// counted once when the plan was built.
static_assert(kF16Item == 8, "an fp16 item is one octet of the group's 8-member padding");
static int expert_items_max(const bitsmoe_plan* p) { return (int)p->max_t1_items; }

// Warps per CTA: every warp owns whole 32-row tiles, so take the count (8..24)
// that leaves the fewest idle warp-tiles, the larger on a tie.
static int choose_warps(int n_rb) {
    int best = 8;
    double best_eff = 0.0;
    for (int nw = 8; nw <= kT1MaxWarps; nw++) {
        const int per = (n_rb + nw - 1) / nw;
        const double eff = (double)n_rb / (double)(per * nw);
        if (eff >= best_eff) {
            best_eff = eff;
            best = nw;
        }
    }
    return best;
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
    P.U = 2 * P.K;
    if (u->dims.d_out != P.d_out || u->dims.rank != P.r || u->dims.d_in != P.d_in) return L;
    if (P.U > kMaxUnits || P.d_in % 8 || P.d_in > 8192 || P.d_pad % kRB) return L;
    P.G = g_num_sms;
    P.n_rb = P.d_pad / kRB;
    const long long q_max = (long long)P.K * (expert_items_max(g) + expert_items_max(u));
    P.items_max = (int)((q_max + P.G - 1) / P.G);
    if (P.items_max > kMaxItems) return L;
    if ((uint64_t)P.G * (uint64_t)std::max<long long>(q_max, 2ll * std::max(P.r, P.d_out) * (P.K + 1)) >= (1ull << 32))
        return L;  // the 32-bit share arithmetic
    if (2ull * kDirEntryBytes * P.E >= (1u << 20)) return L;  // one mbarrier transaction count
    const int im = std::max(1, P.items_max);
    const int phi_rows = (2 * P.r + P.G - 1) / P.G;
    P.sm_x = 0;
    P.sm_dir = align_up(2ull * P.d_in, 128);
    P.sm_phi = align_up(P.sm_dir + 2ull * kDirEntryBytes * P.E, 128);
    P.sm_planes = align_up(P.sm_phi + (uint64_t)phi_rows * P.d_in * 2, 128);
    P.sm_mw = align_up(P.sm_planes + 128ull * P.n_rb * im, 128);
    P.sm_f16 = align_up(P.sm_mw + 256ull * im, 16);
    P.sm_c16 = align_up(P.sm_f16 + 48ull * im, 16);
    P.sm_tab = align_up(P.sm_c16 + 32ull * im, 16);
    P.sm_end = align_up(P.sm_tab + 512ull + 512ull * im, 16);  // + 512: tables realigned in the kernel
    L.smem = P.sm_end;
    if (L.smem + (size_t)g_static_smem > (size_t)g_max_smem) return L;
    L.threads = 32 * choose_warps(P.n_rb);
    // workspace: the launch counter and the zeroing CTAs' tags (a 256-byte head),
    // then the tagged z rows.  All of it persists between calls (a stale z word
    // must never carry a live tag), so other paths work after it.
    L.ws_reserved = 256 + roundup(8ull * 2 * P.r, 256);
    L.ok = true;
    return L;
}

// Bytes at the head of a layer workspace that hold the fused path's
// persistent state: its counters and tagged z rows (0 when it does not apply).
uint64_t layer_fused_t1_reserved(const bitsmoe_plan* g, const bitsmoe_plan* u) {
    T1Layout L = t1_layout(g, u);
    return L.ok ? L.ws_reserved : 0;
}

int layer_forward_fused_t1(const bitsmoe_proj_io** io, const uint16_t* X, const int32_t* ids, const float* gw,
                           void* workspace, uint64_t workspace_bytes, const uint16_t* const* next_phi, int32_t* status,
                           cudaStream_t s, bool* used) {
    *used = false;
    T1Layout L = t1_layout(io[0]->plan, io[1]->plan);
    if (!L.ok || workspace_bytes < L.ws_reserved) return BITSMOE_OK;
    T1Params P = L.P;
    for (int j = 0; j < 2; j++) {
        P.proj[j].blob = (const uint8_t*)io[j]->blob;
        P.proj[j].phi_t = io[j]->phi_t;
        P.proj[j].Z = io[j]->Z;
        P.proj[j].Ye = io[j]->Y_experts;
        P.proj[j].Ysum = io[j]->Y_sum;
    }
    P.next_phi[0] = next_phi ? next_phi[0] : nullptr;
    P.next_phi[1] = next_phi ? next_phi[1] : nullptr;
    P.x = X;
    P.ids = ids;
    P.gw = gw;
    P.status = status;
    uint8_t* ws = (uint8_t*)workspace;
    P.launches = (unsigned long long*)ws;
    P.zero_tags = P.launches + 1;
    P.zbuf = (unsigned long long*)(ws + 256);
    // enough zeroing CTAs that each clears at least kZeroSliceFloats outputs
    const long long n_out = (long long)P.d_out * (2 + (io[0]->Y_experts ? P.K : 0) + (io[1]->Y_experts ? P.K : 0));
    P.n_zero = (int)std::min<long long>({(n_out + kZeroSliceFloats - 1) / kZeroSliceFloats, kMaxZeroCtas, P.G});
    P.n_zero = std::max(P.n_zero, 1);

    cudaError_t e = grant_smem((int)L.smem);
    if (e != cudaSuccess) return set_cuda_error(e);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)P.G);
    cfg.blockDim = dim3((unsigned)L.threads);
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
// cannot allocate device memory.  The scratch (the fused kernel's launch
// counter, its zeroing tags and the tagged z rows of both projections) lives
// in one fixed static device array instead of a caller-provided workspace.
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
    if (head == 0 || head > kNoAllocScratchBytes) return BITSMOE_ESIZE;
    void* scratch = nullptr;
    int rc = noalloc_scratch(&scratch);
    if (rc) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    // The array starts zeroed and every call leaves it ready for the next one
    // (the counter a multiple of the grid, each z word tagged with the launch
    // that wrote it), so it is never cleared: clearing it would restart the
    // tags while z words of earlier calls still carry them.
    bool used = false;
    rc = layer_forward_fused_t1(io, X, topk_ids, gate_w, scratch, head, nullptr, status, s, &used);
    if (rc) return rc;
    return used ? BITSMOE_OK : BITSMOE_ESIZE;
}
