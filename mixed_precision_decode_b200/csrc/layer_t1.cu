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
constexpr int kPhiBars = 4;       // mbarriers over the Phi slice (0 also carries x)
constexpr int kDirBar = kPhiBars;        // the expert directories
constexpr int kPlaneBar = kPhiBars + 1;  // the staged plane words
constexpr int kTagBar = kPhiBars + 2;    // hands this launch's tag to the other warps
constexpr int kPlanBar = kPhiBars + 3;   // the plan is written (the planning warp arrives)
constexpr int kZeroBar = kPhiBars + 4;   // the zeroing warps' stores are done (each arrives)
constexpr int kZBar = kPhiBars + 5;      // the z warps' partial rows are written (each arrives)
constexpr int kCopyBar = kPhiBars + 6;   // the planning warp has issued the plane copies
constexpr int kNumBars = kPhiBars + 7;
constexpr int kMaxRowsPerCta = 32;       // z rows of one CTA: one multi-row warp reduction
constexpr int kZWarps = 8;     // warps that compute the z rows (split along d_in)
constexpr long long kWaitLimitNs = 2000000000LL;  // bounded waits: 2 s, then BITSMOE_ST_TIMEOUT
constexpr int kMaxZeroCtas = 16;       // CTAs that zero the outputs (each publishes a tag)
constexpr int kZeroSliceFloats = 16384;  // outputs zeroed per zeroing CTA, at least
// workspace head: [0] launch counter, [1 .. kMaxZeroCtas] the zeroing CTAs' tags
static_assert(8 * (1 + kMaxZeroCtas) <= 256, "the workspace head is 256 bytes");

struct T1Proj {
    const uint8_t* blob;
    uint64_t blob_bytes;
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
    uint32_t sm_dir, sm_phi, sm_planes, sm_meta, sm_c16, sm_tab, sm_end;
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
// Bounded wait on an mbarrier phase with a short sleep between polls, for waiters
// off the critical path; false on timeout.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > kWaitLimitNs) return false;
        __nanosleep(128);
    }
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
// One routed (projection, slot) pair, as the phases after the plan need it.
struct UnitRef {
    int p, j;  // projection, slot
    float g;   // gate weight
};

// One routed unit's layout, in the planning lane's registers: the groups of its
// expert (storage order; all zero when the id is out of range).
struct UnitRegs {
    uint64_t gbase[kNumGroups];  // byte offset of each group in the blob
    uint32_t n[kNumGroups], np[kNumGroups], pw0[kNumGroups];  // members, padded members, first plane word
    int pw;     // plane words
    int items;  // plane words + octets of fp16 members
};

// d: the unit's directory entry in shared memory, or null for an id out of range.
__device__ __forceinline__ void unit_regs(const uint8_t* d, UnitRegs& R) {
    uint64_t base = 0;
    uint32_t goff[kNumGroups], cnt[kNumGroups];
    if (d) {
        base = *reinterpret_cast<const uint64_t*>(d);
        const uint32_t* go = reinterpret_cast<const uint32_t*>(d + 16);
        const uint16_t* ct = reinterpret_cast<const uint16_t*>(d + 44);
#pragma unroll
        for (int g = 0; g < kNumGroups; g++) {
            goff[g] = go[g];
            cnt[g] = ct[g];
        }
    } else {
#pragma unroll
        for (int g = 0; g < kNumGroups; g++) goff[g] = cnt[g] = 0;
    }
    uint32_t pw = 0;
#pragma unroll
    for (int g = 0; g < kNumGroups; g++) {
        R.n[g] = cnt[g];
        R.np[g] = cnt[g] == 0 ? 0u : (g == 0 ? (cnt[g] + 7u) & ~7u : (cnt[g] + 31u) & ~31u);
        R.pw0[g] = pw;
        R.gbase[g] = base + goff[g];
        if (g > 0) pw += (uint32_t)group_width(g) * (R.np[g] >> 5);
    }
    R.pw = (int)pw;
    R.items = R.pw + (int)((R.n[0] + kF16Item - 1) / kF16Item);
}

// A unit's items, in order: the plane words of its bit-plane groups (group by
// group in storage order; inside a group, word l = jb * W + w is bit plane jb
// of member word w, W words per plane), then the octets of its fp16 members.
// Every CTA takes an equal contiguous share of the concatenation over the
// routed units.  A piece is the part of one group (or of the fp16 octets) of
// one unit that falls in the share: items [l0, l1) of the group, which are
// contiguous both in the blob (planes are [b][W][d_pad], rows fastest) and in
// the CTA's item slots, so one bulk copy stages a piece's plane words.  Its
// member words are the cyclic interval (wstart + k) mod W, k < nw, with
// nw = min(W, l1 - l0): each gets one table slot.
struct Piece {
    const uint8_t* gptr;  // the group's first byte in the blob
    uint32_t np, n;       // padded and stored members of the group
    int16_t u, g;         // unit; group (1..6: bit planes, 0: fp16 octets)
    int16_t l0, l1;       // items [l0, l1) of the group
    int16_t slot0;        // the CTA's item slot of l0
    int16_t tslot0;       // first table slot (bit-plane pieces)
    int16_t nw, wstart;   // member words covered
    int16_t W;            // words per plane (bit-plane pieces)
    int16_t pad_;
};
// A member word (32 members of a group) whose c values and tables this CTA builds.
struct MemberWord {
    const uint8_t* gptr;  // the group's first byte: idx u16[np] | scale u16[np] | amp f32[np] | planes
    uint32_t np;          // padded members of the group
    int16_t p, g, w;
    int16_t nvalid;  // stored members in the word (0..32)
    int16_t zp;      // 1 when this CTA evaluates the word's plane 0 and so owns its zero-point share
    int16_t pad_;
};
// An octet of fp16 members (idx u16[np] | amp f32[np] | w16[np][d_pad]); its
// rows are read in place during the lookups.
struct Octet {
    const uint8_t* gptr;  // the fp16 group's first byte
    uint32_t np;          // padded members of the group
    int16_t l;            // octet index: members 8 l .. 8 l + nf - 1
    int16_t nf;           // stored members in the octet (1..8); 0 for a plane-word item
    int16_t u;
    int16_t pad_;
};
// The items of one unit inside the CTA's share: plane words [i0, ip), fp16
// octets [ip, i1); its member words are table slots [t0, t1).
struct Seg {
    int u, i0, ip, i1, t0, t1;
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
// acc + (low or high fp16 of a) * (the same half of b): a mixed-precision FMA
// (fp16 operands, exact product in fp32, fp32 addend).
template <int HI>
__device__ __forceinline__ float fma_f16x2(uint32_t a, uint32_t b, float acc) {
    float r;
    if (HI)
        asm("{\n .reg .f16 al, ah, bl, bh;\n mov.b32 {al, ah}, %1;\n mov.b32 {bl, bh}, %2;\n"
            " fma.rn.f32.f16 %0, ah, bh, %3;\n}" : "=f"(r) : "r"(a), "r"(b), "f"(acc));
    else
        asm("{\n .reg .f16 al, ah, bl, bh;\n mov.b32 {al, ah}, %1;\n mov.b32 {bl, bh}, %2;\n"
            " fma.rn.f32.f16 %0, al, bl, %3;\n}" : "=f"(r) : "r"(a), "r"(b), "f"(acc));
    return r;
}

// Sums v[i] over the 32 lanes for 8 rows i at once: afterwards every lane l holds
// the sum of row l & 7 (7 halving shuffles, then 2 that add the lane groups).
__device__ __forceinline__ float warp_sum_rows8(float (&v)[8], int lane) {
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1) {
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; i++) {
            const float send = up ? v[i] : v[i + off];
            const float keep = up ? v[i + off] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    float r = v[0];
    r += __shfl_xor_sync(0xffffffffu, r, 8);
    r += __shfl_xor_sync(0xffffffffu, r, 16);
    return r;
}

__global__ void __launch_bounds__(kT1MaxThreads, 1) k_layer_t1(const T1Params P) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t s_bar[kNumBars];
    __shared__ UnitRef s_unit[kMaxUnits];
    __shared__ Piece s_piece[kMaxItems];
    __shared__ MemberWord s_mw[kMaxItems];
    __shared__ Octet s_oct[kMaxItems];
    __shared__ Seg s_seg[kMaxUnits];
    __shared__ uint2 s_desc[kMaxItems];  // plane word: (its tables' shared address, 2^jb bits)
    __shared__ float s_zpmw[kMaxItems];
    __shared__ float s_zpart[kZWarps][32];
    __shared__ int s_ni, s_nmw, s_nseg, s_abort, s_bad;
    __shared__ volatile int s_zto;  // a z poll timed out
    __shared__ uint32_t s_tag;      // this launch's tag (1 .. 2^32 - 1)

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nthreads = blockDim.x, nwarps = nthreads >> 5;
    const int cta = blockIdx.x;
    const int row0 = share_begin(cta, 2 * P.r, P.G), row1 = share_begin(cta + 1, 2 * P.r, P.G);
    const int nrows = row1 - row0;
    const uint32_t row_bytes = (uint32_t)P.d_in * 2;
    // warp roles: 1 plans; 2 .. 2 + nzw - 1 compute the z rows; 0 and the rest zero the outputs
    const int nzw = min(kZWarps, nwarps - 2);
    const bool z_warp = warp >= 2 && warp < 2 + nzw;
    const bool zero_warp = warp != 1 && !z_warp;
    const int n_zero_warps = nwarps - 1 - nzw;

    uint8_t* s_dir = smem + P.sm_dir;  // [projection][expert] directory entries
    uint8_t* s_phi = smem + P.sm_phi;
    uint32_t* s_planes = reinterpret_cast<uint32_t*>(smem + P.sm_planes);  // [item slot][d_pad]
    float* s_c16 = reinterpret_cast<float*>(smem + P.sm_c16);               // [item slot][8]: c of octet members
    // member-word metadata by table slot, 32 members each: idx u16, scale u16, amp f32
    uint16_t* s_midx = reinterpret_cast<uint16_t*>(smem + P.sm_meta);
    uint16_t* s_mscl = s_midx + 32 * P.items_max;
    float* s_mamp = reinterpret_cast<float*>(s_mscl + 32 * P.items_max);
    // tables start on a 512-byte shared-memory boundary: one member word's 8
    // tables are 512 B, so the byte address of a word's tables has a zero low
    // byte and a lookup can splice the entry offset into it with one byte permute
    uint8_t* tab_raw = smem + P.sm_tab;
    float* s_tab = reinterpret_cast<float*>(tab_raw + ((512u - (smem_u32(tab_raw) & 511u)) & 511u));
    const uint32_t tab_sbase = smem_u32(s_tab);

    // ---- launch: one thread initialises the mbarriers and issues the weight copies
    // (expert directories, Phi rows); they are constant, so they go out before the
    // wait for the previous kernel in the stream (programmatic dependent launch) ----
    const bool plan_lane = warp == 1 && lane < P.U;
    if (tid == 0) {
        for (int i = 0; i < kNumBars; i++)
            mbar_init(&s_bar[i], i == kZeroBar ? (uint32_t)n_zero_warps : i == kZBar ? (uint32_t)nzw : 1u);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_abort = 0;
        s_zto = 0;
    }
    __syncthreads();  // the mbarriers are initialised
    if (tid == 0) {
        // both expert directories first: the plan needs them before anything else
        const uint32_t dir_bytes = (uint32_t)P.E * kDirEntryBytes;
        const uint64_t keep = policy_evict_last(), stream = policy_evict_first();
        mbar_expect_tx(&s_bar[kDirBar], 2 * dir_bytes);
        for (int p = 0; p < 2; p++)
            bulk_g2s(s_dir + (size_t)p * dir_bytes, P.proj[p].blob + kHeaderBytes, dir_bytes, &s_bar[kDirBar], keep);
        for (int bi = 0; bi < kPhiBars; bi++) {
            const int ra = row0 + (nrows * bi) / kPhiBars, rbnd = row0 + (nrows * (bi + 1)) / kPhiBars;
            const uint32_t bytes = (uint32_t)(rbnd - ra) * row_bytes;
            mbar_expect_tx(&s_bar[bi], bytes);
            for (int rr = ra; rr < rbnd;) {  // rows are contiguous inside a projection
                const int p = rr / P.r, k = rr - p * P.r;
                const int n = min(rbnd - rr, P.r - k);
                if (in_bounds((uint64_t)(rr - row0 + n) * row_bytes - 1, P.sm_planes - P.sm_phi, P.status) &&
                    in_bounds((uint64_t)(k + n) * P.d_in - 1, (uint64_t)P.r * P.d_in, P.status))
                    bulk_g2s(s_phi + (size_t)(rr - row0) * row_bytes, P.proj[p].phi_t + (size_t)k * P.d_in,
                             (uint32_t)n * row_bytes, &s_bar[bi], stream);
                rr += n;
            }
        }
    }
    // Everything below may read what the previous kernel in the stream wrote (x, the
    // routing, the workspace's counter, tags and z rows, the outputs): wait for it.
    // The next kernel may be launched now; its CTAs start as this kernel's CTAs exit.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int my_id = plan_lane ? P.ids[lane % P.K] : 0;
    const float my_gw = plan_lane ? P.gw[lane % P.K] : 0.0f;
    if (tid == 0) {
        // This launch's tag.  Every launch adds exactly G to the counter (one per
        // CTA, whatever happens later), so before this CTA's addition it holds G
        // times the number of earlier launches n plus fewer than G of this one's.
        // The tag, n mod (2^32 - 1) plus 1, is never 0 (a zero-filled z word) and
        // never that of the launch before.
        const unsigned long long before = atomicAdd(P.launches, 1ull);
        s_tag = (uint32_t)((before / (unsigned long long)P.G) % 0xFFFFFFFFull) + 1u;
        mbar_arrive(&s_bar[kTagBar]);  // publishes s_tag to the other warps
    }

    // ---- the outputs are sums of red.add contributions: the first n_zero CTAs zero
    // them and then publish this launch's tag; every CTA acquires those tags before
    // its first addition ----
    if (cta < P.n_zero && zero_warp) {
        if (!mbar_wait(&s_bar[kTagBar], 0)) s_abort = 1;  // s_tag
        const int zw = warp == 0 ? 0 : warp - 1 - nzw;  // 0 .. n_zero_warps - 1
        const int nys = 2 * P.d_out;
        const int nye0 = P.proj[0].Ye ? P.K * P.d_out : 0, nye1 = P.proj[1].Ye ? P.K * P.d_out : 0;
        const int tot = nys + nye0 + nye1;
        const int a = share_begin(cta, tot, P.n_zero), b = share_begin(cta + 1, tot, P.n_zero);
        for (int i = a + zw * 32 + lane; i < b; i += n_zero_warps * 32) {
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
        // every zeroing warp's stores are ordered before the tag by its release
        // arrival, thread 0's acquiring wait and the cumulative release store
        // (thread 0 wrote s_tag itself)
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_bar[kZeroBar]);
        if (tid == 0) {
            if (mbar_wait(&s_bar[kZeroBar], 0))
                st_release_u64(P.zero_tags + cta, (unsigned long long)s_tag);
            else
                s_abort = 1;
        }
        __syncwarp();
    }

    // ---- the plan of this CTA's share (warp 1): lane u handles routed unit u in its
    // registers, cuts its part of the share into pieces and issues their plane
    // copies itself ----
    if (warp == 1) {
        const bool dir_ok = mbar_wait(&s_bar[kDirBar], 0);
        if (!dir_ok && lane == 0) s_abort = 1;
        const bool is_unit = lane < P.U;
        const int up = is_unit ? lane / P.K : 0, uj = is_unit ? lane - up * P.K : 0;
        const bool valid_e = is_unit && dir_ok && my_id >= 0 && my_id < P.E;
        UnitRegs R;
        unit_regs(valid_e ? s_dir + ((size_t)up * P.E + my_id) * kDirEntryBytes : nullptr, R);
        if (is_unit) s_unit[lane] = UnitRef{up, uj, my_gw};
        const bool bad = __any_sync(0xffffffffu, is_unit && !(my_id >= 0 && my_id < P.E));
        const int items = R.items;  // 0 for a lane past the units or an id out of range
        int incl = items;           // inclusive scan of items over units
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int S = incl - items;  // this unit's first item in the concatenation
        const int Q = __shfl_sync(0xffffffffu, incl, 31);
        const int q0 = share_begin(cta, Q, P.G);
        int ni = share_begin(cta + 1, Q, P.G) - q0;
        if (ni > P.items_max || ni > kMaxItems) {  // the blob's counts disagree with the plan's
            if (lane == 0 && P.status) atomicOr(P.status, BITSMOE_ST_PLANMISMATCH);
            ni = 0;
        }
        const int q1 = q0 + ni;
        // this unit's items inside the share: local indices [a, b)
        const int a = max(q0, S) - S, b = min(q1, S + items) - S;
        const bool live = a < b;
        // pass 1: pieces, member words and staged bytes of this unit
        int npc = 0, ntw = 0;
        uint32_t plane_bytes = 0;
#pragma unroll
        for (int g = 1; g < kNumGroups; g++) {
            const int W = (int)(R.np[g] >> 5), lo = (int)R.pw0[g], hi = lo + group_width(g) * W;
            const int pa = max(a, lo), pb = min(b, hi);
            if (pa < pb) {  // an empty group has lo == hi
                const int nw = min(W, pb - pa);
                npc++;
                ntw += nw;
                plane_bytes += 4u * (uint32_t)P.d_pad * (uint32_t)(pb - pa);
            }
        }
        const int pa16 = max(a, R.pw);
        const bool has16 = pa16 < b;  // fp16 octets [pw, items) meet the share
        if (has16) npc++;
        // one lane arms the plane barrier with the CTA's total before any copy is issued
        uint32_t all_plane_bytes = plane_bytes;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) all_plane_bytes += __shfl_xor_sync(0xffffffffu, all_plane_bytes, o);
        if (lane == 0) mbar_expect_tx(&s_bar[kPlaneBar], all_plane_bytes);
        __syncwarp();
        const uint64_t stream = policy_evict_first();
        const uint8_t* blob = P.proj[up].blob;
        // stage the plane words first (one bulk copy per piece): they are on the critical path
#pragma unroll
        for (int g = 1; g < kNumGroups; g++) {
            const int W = (int)(R.np[g] >> 5), lo = (int)R.pw0[g], hi = lo + group_width(g) * W;
            const int pa = max(a, lo), pb = min(b, hi);
            if (pa < pb &&
                in_bounds((uint64_t)(S + pb - q0) * P.d_pad * 4 - 1, 4ull * P.items_max * P.d_pad, P.status) &&
                in_bounds(R.gbase[g] + 8ull * R.np[g] + 4ull * P.d_pad * (uint64_t)(pb - lo) - 1,
                          P.proj[up].blob_bytes, P.status))
                bulk_g2s(s_planes + (size_t)(S + pa - q0) * P.d_pad,
                         blob + R.gbase[g] + 8ull * R.np[g] + 4ull * P.d_pad * (uint64_t)(pa - lo),
                         4u * (uint32_t)P.d_pad * (uint32_t)(pb - pa), &s_bar[kPlaneBar], stream);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_bar[kCopyBar]);  // the z warps may start
        int pinc = npc, tinc = ntw;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, pinc, o), w = __shfl_up_sync(0xffffffffu, tinc, o);
            if (lane >= o) {
                pinc += v;
                tinc += w;
            }
        }
        const int npieces = __shfl_sync(0xffffffffu, pinc, 31), ntab = __shfl_sync(0xffffffffu, tinc, 31);
        const unsigned lt = (1u << lane) - 1u;
        const unsigned blive = __ballot_sync(0xffffffffu, live);
        // pass 2a: write the pieces
        {
            int k = pinc - npc, t = tinc - ntw;
#pragma unroll
            for (int g = 1; g < kNumGroups; g++) {
                const int W = (int)(R.np[g] >> 5), lo = (int)R.pw0[g], hi = lo + group_width(g) * W;
                const int pa = max(a, lo), pb = min(b, hi);
                if (pa < pb) {
                    const int nw = min(W, pb - pa);
                    const int l0 = pa - lo;
                    int wstart = 0;
                    if (nw < W) {
                        wstart = l0;
                        while (wstart >= W) wstart -= W;  // l0 mod W (l0 < 8 W)
                    }
                    Piece X;
                    X.gptr = blob + R.gbase[g];
                    X.np = R.np[g];
                    X.n = R.n[g];
                    X.u = (int16_t)lane;
                    X.g = (int16_t)g;
                    X.l0 = (int16_t)l0;
                    X.l1 = (int16_t)(pb - lo);
                    X.slot0 = (int16_t)(S + pa - q0);
                    X.tslot0 = (int16_t)t;
                    X.nw = (int16_t)nw;
                    X.wstart = (int16_t)wstart;
                    X.W = (int16_t)W;
                    X.pad_ = 0;
                    if (in_bounds(k, kMaxItems, P.status) && in_bounds(t + nw - 1, (uint64_t)P.items_max, P.status))
                        s_piece[k] = X;
                    k++;
                    t += nw;
                }
            }
            if (has16) {
                Piece X;
                X.gptr = blob + R.gbase[0];
                X.np = R.np[0];
                X.n = R.n[0];
                X.u = (int16_t)lane;
                X.g = 0;
                X.l0 = (int16_t)(pa16 - R.pw);
                X.l1 = (int16_t)(b - R.pw);
                X.slot0 = (int16_t)(S + pa16 - q0);
                X.tslot0 = (int16_t)t;
                X.nw = X.wstart = X.W = X.pad_ = 0;
                if (in_bounds(k, kMaxItems, P.status)) s_piece[k] = X;
            }
        }
        if (live) {
            Seg G;
            G.u = lane;
            G.i0 = S + a - q0;
            G.ip = S + max(a, min(b, R.pw)) - q0;
            G.i1 = S + b - q0;
            G.t0 = tinc - ntw;
            G.t1 = tinc;
            s_seg[__popc(blive & lt)] = G;
        }
        __syncwarp();  // every lane has written its pieces
        if (lane == 0) {
            s_ni = ni;
            s_nmw = ntab;
            s_nseg = __popc(blive);
            s_bad = bad;
        }
        // item descriptors: lane i finds the piece of item slot i
        if (lane < ni) {
            int k = 0;
            while (k + 1 < npieces && s_piece[k + 1].slot0 <= lane) k++;
            const Piece X = s_piece[k];
            const int l = X.l0 + (lane - X.slot0);
            Octet O;
            O.gptr = X.gptr;
            O.np = X.np;
            O.l = 0;
            O.nf = 0;
            O.u = X.u;
            O.pad_ = 0;
            if (X.g > 0) {
                int jb = 0, w = l;
                while (w >= X.W) {  // l = jb * W + w, jb < 8
                    w -= X.W;
                    jb++;
                }
                int t = w - X.wstart;
                if (t < 0) t += X.W;
                if (!in_bounds(X.tslot0 + t, (uint64_t)P.items_max, P.status)) t = -X.tslot0;  // slot 0: a wrong sum, no stray access
                s_desc[lane] = make_uint2(tab_sbase + 512u * (uint32_t)(X.tslot0 + t), __float_as_uint((float)(1u << jb)));
            } else {
                O.l = (int16_t)l;
                O.nf = (int16_t)min(kF16Item, (int)X.n - kF16Item * l);
                s_desc[lane] = make_uint2(0u, 0u);
            }
            s_oct[lane] = O;
        }
        // member words: lane t finds the bit-plane piece of table slot t
        for (int t = lane; t < ntab; t += 32) {
            int k = 0;
            while (k + 1 < npieces && s_piece[k + 1].tslot0 <= t) k++;
            const Piece X = s_piece[k];
            int w = X.wstart + (t - X.tslot0);
            if (w >= X.W) w -= X.W;
            MemberWord M;
            M.gptr = X.gptr;
            M.np = X.np;
            M.p = (int16_t)(X.u / P.K);
            M.g = X.g;
            M.w = (int16_t)w;
            M.nvalid = (int16_t)max(0, min(32, (int)X.n - 32 * w));
            M.zp = (int16_t)(w >= X.l0 && w < X.l1);  // plane 0 of word w is item w of the group
            M.pad_ = 0;
            s_mw[t] = M;
        }
        __syncwarp();  // the plan's shared-memory writes of every lane precede lane 0's release
        if (lane == 0) mbar_arrive(&s_bar[kPlanBar]);
        // the zeroing CTAs' tags (bounded waits), while the other warps compute z
        const bool tag_ok = mbar_wait(&s_bar[kTagBar], 0);
        if (lane < P.n_zero && (!tag_ok || !tag_wait(P.zero_tags + lane, (unsigned long long)s_tag))) s_abort = 1;
        __syncwarp();
    } else if (!z_warp) {
        // the plan (bounded wait with back-off: these warps have nothing else to do,
        // and polling would take issue slots from the planning and z warps)
        if (!mbar_wait_sleep(&s_bar[kPlanBar], 0)) s_abort = 1;
        // the metadata (idx, scale, amp) of every member word of the plan into shared
        // memory, split over these warps (warp 0 and those after the z warps): one
        // coalesced load per array and word
        const int nmw_ = s_nmw, nlw = n_zero_warps, lw = warp == 0 ? 0 : warp - 1 - nzw;
        for (int m = lw; m < nmw_; m += nlw) {
            const MemberWord M = s_mw[m];
            const int k = 32 * M.w + lane;  // member of the group (padding members carry zeros)
            if (!in_bounds(m, (uint64_t)P.items_max, P.status) || !in_bounds(k, M.np, P.status)) continue;
            s_midx[32 * m + lane] = reinterpret_cast<const uint16_t*>(M.gptr)[k];
            s_mscl[32 * m + lane] = reinterpret_cast<const uint16_t*>(M.gptr + 2ull * M.np)[k];
            s_mamp[32 * m + lane] = reinterpret_cast<const float*>(M.gptr + 4ull * M.np)[k];
        }
    }



    // ---- z rows of this CTA, split along d_in over the z warps: lane l of z warp zw
    // owns 16-byte chunks l + 32 (zw + nzw m) of x (in registers) and accumulates
    // every row's partial dot product over them; a multi-row warp reduction and a sum
    // over the z warps give the rows, each published with this launch's tag ----
    if (z_warp) {
        const int zw = warp - 2;
        // The z arithmetic (fp16 products, issue- and conversion-bound) starts once the
        // planning warp has issued the plane copies, which everything after z waits for.
        bool ok = mbar_wait_sleep(&s_bar[kCopyBar], 0);
        ok = ok && (nrows == 0 || mbar_wait(&s_bar[kTagBar], 0));
        const unsigned long long tag_hi = (unsigned long long)s_tag << 32;
        const int nch = P.d_in / 8;
        const uint4* xv = reinterpret_cast<const uint4*>(P.x);  // 16-byte chunks of x
        const uint4 xc0 = lane + 32 * zw < nch ? xv[lane + 32 * zw] : make_uint4(0, 0, 0, 0);  // this lane's first
        // chunk bi holds rows [nrows bi / 4, nrows (bi + 1) / 4): at most 8 of the at most
        // kMaxRowsPerCta rows.  Per chunk: 8 row partials per lane, an 8-row warp reduction
        // (lane l ends with row l & 7), and the warp's row sums into s_zpart.
        for (int bi = 0; bi < kPhiBars; bi++) {
            const int ra = (nrows * bi) / kPhiBars, rn = (nrows * (bi + 1)) / kPhiBars - ra;
            if (!mbar_wait(&s_bar[bi], 0)) ok = false;
            if (rn == 0) continue;
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; i++) acc[i] = 0.0f;
            for (int c = lane + 32 * zw; c < nch; c += 32 * nzw) {
                const uint4 xc = c == lane + 32 * zw ? xc0 : xv[c];
                const uint4* rp = reinterpret_cast<const uint4*>(s_phi + (size_t)ra * row_bytes) + c;
                // rows in two groups of 4: the 4 loads first (rows past the chunk repeat its
                // last row; their sums are never stored), then the FMAs interleaved over the
                // 4 independent rows
#pragma unroll
                for (int g4 = 0; g4 < 8; g4 += 4) {
                    uint4 v[4];
#pragma unroll
                    for (int i = 0; i < 4; i++) v[i] = rp[(size_t)min(g4 + i, rn - 1) * (row_bytes / 16)];
#pragma unroll
                    for (int i = 0; i < 4; i++) acc[g4 + i] = fma_f16x2<0>(v[i].x, xc.x, acc[g4 + i]);
#pragma unroll
                    for (int i = 0; i < 4; i++) acc[g4 + i] = fma_f16x2<1>(v[i].x, xc.x, acc[g4 + i]);
#pragma unroll
                    for (int i = 0; i < 4; i++) acc[g4 + i] = fma_f16x2<0>(v[i].y, xc.y, acc[g4 + i]);
#pragma unroll
                    for (int i = 0; i < 4; i++) acc[g4 + i] = fma_f16x2<1>(v[i].y, xc.y, acc[g4 + i]);
#pragma unroll
                    for (int i = 0; i < 4; i++) acc[g4 + i] = fma_f16x2<0>(v[i].z, xc.z, acc[g4 + i]);
#pragma unroll
                    for (int i = 0; i < 4; i++) acc[g4 + i] = fma_f16x2<1>(v[i].z, xc.z, acc[g4 + i]);
#pragma unroll
                    for (int i = 0; i < 4; i++) acc[g4 + i] = fma_f16x2<0>(v[i].w, xc.w, acc[g4 + i]);
#pragma unroll
                    for (int i = 0; i < 4; i++) acc[g4 + i] = fma_f16x2<1>(v[i].w, xc.w, acc[g4 + i]);
                }
            }
            const float part = warp_sum_rows8(acc, lane);
            if (lane < rn) s_zpart[zw][ra + lane] = part;
        }
        if (nrows > 0) {  // at most kMaxRowsPerCta rows (the host checks it)
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_bar[kZBar]);  // releases this warp's partial rows
            if (zw == 0) {
                if (!mbar_wait(&s_bar[kZBar], 0)) ok = false;
                if (ok && lane < nrows && in_bounds(row0 + lane, 2ull * P.r, P.status)) {
                    float z = 0.0f;
                    for (int w = 0; w < nzw; w++) z += s_zpart[w][lane];
                    const int rr = row0 + lane, p = rr / P.r, k = rr - p * P.r;
                    st_relaxed_u64(P.zbuf + rr, tag_hi | __float_as_uint(z));
                    if (P.proj[p].Z) P.proj[p].Z[k] = z;
                }
            }
        }
        if (!ok) s_abort = 1;
    }
    if (tid == 0) {
        // every bulk copy into this CTA's shared memory lands before it can exit
        for (int bi = 0; bi < kPhiBars; bi++)
            if (!mbar_wait(&s_bar[bi], 0)) s_abort = 1;
        if (!mbar_wait(&s_bar[kPlaneBar], 0)) s_abort = 1;  // the staged planes
        if (s_bad && cta == 0 && P.status) atomicOr(P.status, BITSMOE_ST_BADEXPERT);
        // This CTA's reads from HBM are done: while the experts are evaluated, pull
        // its rows of the next layer's Phi into L2 for the next call.
        if (!s_abort && P.next_phi[0] && P.next_phi[1])
            for (int rr = row0; rr < row1;) {
                const int p = rr / P.r, k = rr - p * P.r;
                const int n = min(row1 - rr, P.r - k);
                bulk_prefetch_l2(P.next_phi[p] + (size_t)k * P.d_in, (uint32_t)n * row_bytes);
                rr += n;
            }
    }
    __syncwarp();
    __syncthreads();
    if (s_abort) {
        if (tid == 0 && P.status) atomicOr(P.status, BITSMOE_ST_TIMEOUT);
        return;
    }
    const int ni = s_ni, nseg = s_nseg;
    const uint32_t tag = s_tag;

    // ---- c_k = a_k s_k z_k, the tables and the zero-point share: a warp per member word ----
    const int nmw = s_nmw;
    for (int m = warp; m < nmw; m += nwarps) {
        const MemberWord M = s_mw[m];
        const int k = s_midx[32 * m + lane];
        float c = 0.0f;
        if (lane < M.nvalid && k < P.r && in_bounds(M.p * P.r + k, 2ull * P.r, P.status))
            c = s_mamp[32 * m + lane] * __half2float(__ushort_as_half(s_mscl[32 * m + lane])) *
                z_poll(P.zbuf + M.p * P.r + k, tag, &s_zto);
        // entry e of table tb = the sum of c over the set bits of e (members 4 tb .. 4 tb + 3)
        const int e = lane & 15;
#pragma unroll
        for (int qq = 0; qq < 4; qq++) {
            const int tb = (lane >> 4) + 2 * qq;
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
        const Octet O = s_oct[i];
        if (!O.nf) continue;
        float c = 0.0f;
        if (m < O.nf) {
            const int k = reinterpret_cast<const uint16_t*>(O.gptr)[kF16Item * O.l + m];
            if (k < P.r)
                c = reinterpret_cast<const float*>(O.gptr + 2ull * O.np)[kF16Item * O.l + m] *
                    z_poll(P.zbuf + s_unit[O.u].p * P.r + k, tag, &s_zto);
        }
        s_c16[kF16Item * i + m] = c;
    }
    __syncwarp();
    __syncthreads();
    if (s_zto) {
        if (tid == 0 && P.status) atomicOr(P.status, BITSMOE_ST_TIMEOUT);
        return;
    }

    // ---- lookups: warps own 32-row tiles; a segment's rows go to Y_e and, times g, to Y_sum ----
    for (int s = 0; s < nseg; s++) {
        const Seg S = s_seg[s];
        const UnitRef U = s_unit[S.u];
        const int p = U.p;
        float* ye = P.proj[p].Ye ? P.proj[p].Ye + (size_t)U.j * P.d_out : nullptr;
        float* ys = P.proj[p].Ysum;
        const float gj = U.g;
        // this CTA's zero-point share of the unit (its member words are slots [t0, t1), at most 32)
        const float zps = warp_sum(S.t0 + lane < S.t1 ? s_zpmw[S.t0 + lane] : 0.0f);
        for (int t = warp; t < P.n_rb; t += nwarps) {
            const uint32_t* pl = s_planes + t * kRB + lane;  // [item slot][d_pad]
            float acc = 0.0f;
#pragma unroll 4
            for (int i = S.i0; i < S.ip; i++) {
                if (!in_bounds((uint64_t)i * P.d_pad + t * kRB + lane, (uint64_t)P.items_max * P.d_pad, P.status)) break;
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
                const Octet O = s_oct[i];
                const uint16_t* w16 = reinterpret_cast<const uint16_t*>(O.gptr + 6ull * O.np) +
                                      (size_t)kF16Item * O.l * P.d_pad;
                for (int m = 0; m < O.nf; m++)
                    acc = fmaf(s_c16[kF16Item * i + m], __half2float(__ushort_as_half(w16[(size_t)m * P.d_pad + row])),
                               acc);
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

// Limits of the current device that the launch shape depends on, looked up once per
// device (a process may drive GPUs of different SM counts).
struct DeviceInfo {
    int num_sms, max_smem, static_smem;
};

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

static std::mutex g_devinfo_mu;
static DeviceInfo g_devinfo[kMaxDevices];
static bool g_devinfo_ok[kMaxDevices];

static bool device_info(DeviceInfo* out) {
    int dev;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lock(g_devinfo_mu);
    if (!g_devinfo_ok[dev]) {
        DeviceInfo d{};
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
        if (cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return false;
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, k_layer_t1) != cudaSuccess) return false;
        d.static_smem = (int)fa.sharedSizeBytes;
        g_devinfo[dev] = d;
        g_devinfo_ok[dev] = true;
    }
    *out = g_devinfo[dev];
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
    DeviceInfo dv;
    if (!device_info(&dv)) return L;
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
    P.G = dv.num_sms;
    P.n_rb = P.d_pad / kRB;
    const long long q_max = (long long)P.K * (expert_items_max(g) + expert_items_max(u));
    P.items_max = (int)((q_max + P.G - 1) / P.G);
    if (P.items_max > kMaxItems) return L;
    if ((uint64_t)P.G * (uint64_t)std::max<long long>(q_max, 2ll * std::max(P.r, P.d_out) * (P.K + 1)) >= (1ull << 32))
        return L;  // the 32-bit share arithmetic
    if (2ull * kDirEntryBytes * P.E >= (1u << 20)) return L;  // one mbarrier transaction count
    // the staged planes of one CTA are one mbarrier transaction count
    if (4ull * P.d_pad * P.items_max >= (1u << 20)) return L;
    const int im = std::max(1, P.items_max);
    const int phi_rows = (2 * P.r + P.G - 1) / P.G;
    if (phi_rows > kMaxRowsPerCta) return L;  // one multi-row warp reduction of z per CTA
    P.sm_dir = 0;
    P.sm_phi = align_up(P.sm_dir + 2ull * kDirEntryBytes * P.E, 128);
    P.sm_planes = align_up(P.sm_phi + (uint64_t)phi_rows * P.d_in * 2, 128);
    P.sm_meta = align_up(P.sm_planes + 128ull * P.n_rb * im, 16);
    P.sm_c16 = align_up(P.sm_meta + 256ull * im, 16);
    P.sm_tab = align_up(P.sm_c16 + 32ull * im, 16);
    P.sm_end = align_up(P.sm_tab + 512ull + 512ull * im, 16);  // + 512: tables realigned in the kernel
    L.smem = P.sm_end;
    if (L.smem + (size_t)dv.static_smem > (size_t)dv.max_smem) return L;
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
        P.proj[j].blob_bytes = io[j]->plan->blob_bytes;
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
    // Programmatic dependent launch: consecutive calls in a stream overlap the next
    // launch with this one's tail.  Every CTA must be resident at once (the z rows and
    // zeroing tags are exchanged between CTAs): one CTA per SM, which the shared-memory
    // size enforces, and every wait between CTAs is bounded (BITSMOE_ST_TIMEOUT).
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
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
