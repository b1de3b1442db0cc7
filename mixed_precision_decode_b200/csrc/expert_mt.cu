// expert_mt.cu -- routed expert forward for any number of tokens: the
// width-grouped bit planes of one expert, evaluated bit-serially for every
// token routed to it (BitsMoE study-note page, Methodology: W_e x =
// P_e A_e (Phi^T x); Execution: bit planes grouped by width):
//   y_{t,i} = sum_b sum_j 2^j sum_{k in G_b} c_{k,t} bit_{k,j,i}
//             - sum_b (2^b - 1)/2 sum_{k in G_b} c_{k,t}
//             + sum_{k in G_16} a_k z_{t,k} w16_{k,i},        c_{k,t} = a_k s_k z_{t,k}.
//
// Two kernels.  k_cvals forms, once per routed (token, slot) pair, c for every
// member of the pair's expert (a_k z_{t,k} for the fp16 members) and the
// pair's zero-point total, into a workspace buffer.  k_expert_mt then runs one
// CTA per (routed expert, range of up to 4 tiles of 32 rows), 16 warps, two
// CTAs per SM: it stages its tiles of every plane word in shared memory with
// 16-byte cp.async pieces from every thread (a plane word gives a CTA only
// 128 B per tile, too little for a bulk copy apiece) and the c rows of up to
// four of the expert's tokens with one bulk copy each.  Each warp takes a contiguous
// range of the expert's member words (balanced by plane words) and, per word,
// builds in its own 2 KB of shared memory the word's 16-entry subset-sum
// tables whose entries are token PAIRS (float2), from broadcast 16-byte loads
// of the staged c rows, then looks up
// every plane word of the member word for every tile: one conflict-free 8-byte
// shared load per 4-member nibble and two tokens, a lane per row.  The loop
// needs no CTA barrier; the warps' partial sums are added in warp order at the
// end, so the outputs do not depend on timing.
#include <algorithm>

#include "common.cuh"

namespace bitsmoe {

constexpr int kMtThreads = 512;  // 16 warps; two CTAs share an SM
constexpr int kMtWarps = kMtThreads / 32;
constexpr int kMtTok = 4;           // tokens per group
constexpr int kMtPairs = kMtTok / 2;
constexpr int kMtMaxTiles = 4;      // 32-row tiles per CTA, at most
constexpr uint32_t kMtBuildCost = 5;  // a member word's table build, in lookups of one plane word, tile and pair
constexpr int kCvThreads = 1024;
constexpr int kCvPer = 2;          // members of a c row per thread and pass
constexpr long long kMtWaitNs = 2000000000LL;

struct MtParams {
    const uint8_t* blob;
    uint64_t blob_bytes;
    uint32_t stage_words;  // words of the staging buffer
    uint32_t c_floats;     // floats of the c rows' buffer
    int n_pairs;           // T * K: rows of Y_e
    RouteWS rw;
    float* Ye;
    int32_t* status;
    int K, d_out, d_pad, n_tiles;
    int tiles_per_cta;  // 1, 2 or 4
    uint32_t sm_stage, sm_c, sm_tab;
};

__device__ __forceinline__ uint32_t mt_smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ long long mt_globaltimer() {
    long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mt_mbar_init(uint64_t* bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mt_smem_u32(bar)));
}
__device__ __forceinline__ void mt_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mt_smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mt_mbar_wait(uint64_t* bar, uint32_t parity) {
    const long long t0 = mt_globaltimer();
    for (;;) {
        uint32_t ok;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(ok)
            : "r"(mt_smem_u32(bar)), "r"(parity)
            : "memory");
        if (ok) return true;
        if (mt_globaltimer() - t0 > kMtWaitNs) return false;
    }
}
__device__ __forceinline__ void mt_bulk(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     mt_smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(mt_smem_u32(bar))
                 : "memory");
}
// 8-byte shared load (a token pair) at a 32-bit shared address plus a constant.
template <int OFF>
__device__ __forceinline__ float2 mt_lds2(uint32_t addr) {
    float2 v;
    asm("ld.shared.v2.f32 {%0, %1}, [%2+%3];" : "=f"(v.x), "=f"(v.y) : "r"(addr), "n"(OFF));
    return v;
}
__device__ __forceinline__ float2 f2add(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
// 4-byte shared load (one token) at a 32-bit shared address plus a constant.
template <int OFF>
__device__ __forceinline__ float mt_lds1(uint32_t addr) {
    float v;
    asm("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(OFF));
    return v;
}

// Warp 0 (every lane): records the token group's pairs (lane u holds the pair of
// token u, or -1 past the group's nt tokens) and their zero-point totals, and
// issues one bulk copy of each pair's c row into row u of s_c, all on one phase
// of bar.  In the checked build a copy that would leave its buffer is skipped
// and not counted in the phase's bytes.
__device__ __forceinline__ void mt_issue_group(const MtParams& P, int pr, int nt, uint32_t members, int lane,
                                               int* s_pair, float* s_zp, float* s_c, uint64_t* bar) {
    const bool ok = lane < nt && pr >= 0 && members > 0 &&
                    in_bounds((uint64_t)(lane + 1) * members - 1, P.c_floats, P.status) &&
                    in_bounds((uint64_t)pr, (uint64_t)P.n_pairs, P.status);
    const uint32_t okm = __ballot_sync(0xffffffffu, ok);
    if (lane == 0) mt_expect_tx(bar, 4u * members * (uint32_t)__popc(okm));
    __syncwarp();
    if (ok) mt_bulk(s_c + (size_t)lane * members, P.rw.cvals + (size_t)pr * P.rw.ldc, 4u * members, bar);
    if (lane < kMtTok) {
        s_pair[lane] = lane < nt ? pr : -1;
        s_zp[lane] = ok ? P.rw.zp[pr] : 0.0f;
    }
}

// ---------------------------------------------------------------------------
// c values: one CTA per routed pair q = t * K + j
// ---------------------------------------------------------------------------
// C[q][m] over the member slots m of the pair's expert, groups in storage
// order (fp16 first), each padded to its np: a_k s_k z_{t,k} for the bit-plane
// members, a_k z_{t,k} for the fp16 members, 0 for padding (and for an index
// k >= r, which only a corrupt blob holds).  zp[q] = sum over the bit-plane
// groups of (2^b - 1)/2 sum_k c_k.
__global__ void __launch_bounds__(kCvThreads) k_cvals(const uint8_t* __restrict__ blob, const float* __restrict__ Z,
                                                      const int32_t* __restrict__ ids, int K, int E, int r,
                                                      RouteWS rw) {
    __shared__ float s_red[kCvThreads / 32];
    __shared__ uint32_t start[kNumGroups + 1], s_n[kNumGroups];  // first c slot and members of each group
    __shared__ const uint8_t* s_gm[kNumGroups];                  // each group's metadata
    const int q = blockIdx.x, t = q / K, tid = threadIdx.x;
    const int e = ids[q];
    if (e < 0 || e >= E) return;  // the routing groups leave this pair out
    if (tid == 0) {
        const DirEntry d = read_dir(blob, e);
        start[0] = 0;
        for (int g = 0; g < kNumGroups; g++) {
            start[g + 1] = start[g] + (uint32_t)group_members_padded(group_width(g), d.count[g]);
            s_n[g] = d.count[g];
            s_gm[g] = blob + d.base + d.goff[g];
        }
    }
    __syncthreads();
    float* Cq = rw.cvals + (size_t)q * rw.ldc;
    const float* zt = Z + (size_t)t * r;
    float zsum = 0.0f;
    // kCvPer members a thread per pass; every load of a pass is issued before its z loads
    for (uint32_t m0 = 0; m0 < start[kNumGroups]; m0 += kCvThreads * kCvPer) {
        int kk[kCvPer], gg[kCvPer];
        float f[kCvPer];  // a_k s_k (bit-plane member) or a_k (fp16 member); 0 for padding
#pragma unroll
        for (int v = 0; v < kCvPer; v++) {
            const uint32_t m = m0 + (uint32_t)tid + (uint32_t)v * kCvThreads;
            int g = 0;
#pragma unroll
            for (int h = 1; h < kNumGroups; h++) g += m >= start[h] ? 1 : 0;
            gg[v] = m < start[kNumGroups] ? g : -1;
            kk[v] = r;
            f[v] = 0.0f;
            if (gg[v] >= 0) {
                const uint32_t ml = m - start[g], np = start[g + 1] - start[g];
                if (ml < s_n[g]) {
                    const uint8_t* gm = s_gm[g];
                    kk[v] = reinterpret_cast<const uint16_t*>(gm)[ml];
                    if (group_width(g) == 16) {
                        f[v] = reinterpret_cast<const float*>(gm + 2ull * np)[ml];
                    } else {
                        const uint16_t sh = reinterpret_cast<const uint16_t*>(gm + 2ull * np)[ml];
                        f[v] = reinterpret_cast<const float*>(gm + 4ull * np)[ml] * __half2float(__ushort_as_half(sh));
                    }
                }
            }
        }
#pragma unroll
        for (int v = 0; v < kCvPer; v++) {
            if (gg[v] < 0) continue;
            const float c = kk[v] < r ? f[v] * __ldg(zt + kk[v]) : 0.0f;
            Cq[m0 + (uint32_t)tid + (uint32_t)v * kCvThreads] = c;
            if (gg[v] > 0) zsum += 0.5f * (float)((1 << group_width(gg[v])) - 1) * c;
        }
    }
    for (int o = 16; o > 0; o >>= 1) zsum += __shfl_xor_sync(0xffffffffu, zsum, o);
    if ((tid & 31) == 0) s_red[tid >> 5] = zsum;
    __syncthreads();
    if (tid == 0) {
        float sum = 0.0f;
        for (int w = 0; w < kCvThreads / 32; w++) sum += s_red[w];
        rw.zp[q] = sum;
    }
}

// ---------------------------------------------------------------------------
// expert evaluation: one CTA per (routed expert, range of tiles)
// ---------------------------------------------------------------------------
// Per-expert shape of the staged data.
struct MtExpert {
    uint32_t n[kNumGroups], np[kNumGroups], W[kNumGroups];
    uint32_t stage_off[kNumGroups];  // word offset of the group's tiles in the staging buffer
    uint32_t c_off[kNumGroups];      // member offset of the group in a c row
    uint64_t gbase[kNumGroups];      // byte offset of the group in the blob
    uint32_t members;                // padded members of all groups: the length of a c row
    uint32_t plane_words;            // b W summed over the bit-plane groups
};

__global__ void __launch_bounds__(kMtThreads) k_expert_mt(const MtParams P) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint64_t s_cbar;  // the c rows of a token group (one phase per group)
    __shared__ MtExpert s_ex;
    __shared__ int s_pair[kMtTok], s_fail;
    __shared__ float s_zp[kMtTok];
    __shared__ int s_wbeg[kMtWarps + 1];  // member words of each warp (a contiguous range)

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int slot = blockIdx.x;
    if (slot >= *P.rw.nactive) return;
    const int e = P.rw.active[slot];
    const int p0 = P.rw.start[e], p1 = P.rw.start[e + 1];
    const int tile0 = blockIdx.y * P.tiles_per_cta;
    const int ntl = min(P.tiles_per_cta, P.n_tiles - tile0);
    if (ntl <= 0) return;

    uint32_t* s_stage = reinterpret_cast<uint32_t*>(smem + P.sm_stage);
    float* s_c = reinterpret_cast<float*>(smem + P.sm_c);  // [token][members]
    // each warp's token-pair tables: a 2048-byte block (pair 0, then pair 1) of
    // 8 nibble tables x 16 float2, on a 1024-byte boundary
    const uint32_t tab_raw = mt_smem_u32(smem + P.sm_tab);
    const uint32_t tab_s = (tab_raw + 1023u) & ~1023u;
    float2* s_tab = reinterpret_cast<float2*>(smem + P.sm_tab + (tab_s - tab_raw));
    float2* my_tab = s_tab + (size_t)warp * 256;
    const uint32_t my_tab_s = tab_s + 2048u * (uint32_t)warp;
    float* s_part = reinterpret_cast<float*>(s_tab);  // reused after the lookups: [warp][tile][32][kMtTok]

    // ---- warp 0: the first token group's c rows are requested first (the pair ids
    // load while lane 0 reads the directory), then lane 0 lays out the expert ----
    if (warp == 0) {
        const int nt0 = min(kMtTok, p1 - p0);
        const int pr0 = lane < nt0 ? P.rw.pairs[p0 + lane] : -1;
        DirEntry d;
        uint32_t members0 = 0;
        if (lane == 0) {
            d = read_dir(P.blob, e);
            for (int g = 0; g < kNumGroups; g++) members0 += (uint32_t)group_members_padded(group_width(g), d.count[g]);
            s_fail = 0;
            mt_mbar_init(&s_cbar);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        members0 = __shfl_sync(0xffffffffu, members0, 0);
        mt_issue_group(P, pr0, nt0, members0, lane, s_pair, s_zp, s_c, &s_cbar);
        if (lane == 0) {
            uint32_t so = 0, co = 0, pw = 0, pwords = 0;
            for (int g = 0; g < kNumGroups; g++) {
                const int b = group_width(g);
                s_ex.n[g] = d.count[g];
                s_ex.np[g] = (uint32_t)group_members_padded(b, d.count[g]);
                s_ex.W[g] = b == 16 ? 0 : s_ex.np[g] / 32;
                s_ex.stage_off[g] = so;
                s_ex.c_off[g] = co;
                s_ex.gbase[g] = d.base + d.goff[g];
                if (b != 16) {
                    so += (uint32_t)ntl * b * s_ex.W[g] * 32;
                    pw += (uint32_t)s_ex.W[g] * (2u * (uint32_t)b * (uint32_t)ntl + kMtBuildCost);
                    pwords += (uint32_t)b * s_ex.W[g];
                }
                co += s_ex.np[g];
            }
            s_ex.members = co;
            // member words (in group order) shared out over the warps by cost (the
            // lookups of b planes x ntl tiles x 2 token pairs, plus one table build):
            // warp v takes the words whose cost starts in [pw v / warps, pw (v + 1) / warps)
            int wv = 0;
            uint32_t acc_pw = 0, word = 0;
            s_wbeg[0] = 0;
            for (int g = 1; g < kNumGroups; g++) {
                const uint32_t b = (uint32_t)group_width(g);
                for (uint32_t w = 0; w < s_ex.W[g]; w++, word++) {
                    while (wv < kMtWarps - 1 && (uint64_t)acc_pw * kMtWarps >= (uint64_t)pw * (wv + 1)) s_wbeg[++wv] = (int)word;
                    acc_pw += 2u * b * (uint32_t)ntl + kMtBuildCost;
                }
            }
            while (wv < kMtWarps) s_wbeg[++wv] = (int)word;
            s_ex.plane_words = pwords;
        }
    }
    __syncthreads();  // s_ex, the word ranges and the mbarriers are ready
    // ---- stage this CTA's rows of every plane word of the expert: plane word q of
    // group g holds rows [32 tile0, 32 (tile0 + ntl)) contiguously in the blob ([b][W][d_pad],
    // rows fastest); they are staged as [b][W][32 ntl], by every thread in 16-byte
    // pieces (cp.async: a CTA's plane words are too many, and each too short, for
    // one bulk copy apiece) ----
    {
        const uint32_t per_word = 8u * (uint32_t)ntl;  // 16-byte pieces of one plane word's rows
        const uint32_t total = s_ex.plane_words * per_word;
        int g = 1;
        uint32_t qg = 0;  // first plane word of group g
        for (uint32_t i = tid; i < total; i += kMtThreads) {
            const uint32_t q = i / per_word, piece = i - q * per_word;
            while (g < kNumGroups && q >= qg + (uint32_t)group_width(g) * s_ex.W[g]) {
                qg += (uint32_t)group_width(g) * s_ex.W[g];
                g++;
            }
            if (g >= kNumGroups) break;  // only past the expert's plane words (never, if the counts agree)
            const uint8_t* src = P.blob + s_ex.gbase[g] + 8ull * s_ex.np[g] +
                                 4ull * ((uint64_t)(q - qg) * (uint64_t)P.d_pad + 32ull * tile0) + 16ull * piece;
            const uint32_t dst = mt_smem_u32(s_stage + s_ex.stage_off[g] + (q - qg) * 32u * ntl + 4u * piece);
            if (!in_bounds(s_ex.stage_off[g] + (q - qg) * 32u * ntl + 4u * piece + 3u, P.stage_words, P.status) ||
                !in_bounds((uint64_t)(src - P.blob) + 15u, P.blob_bytes, P.status))
                continue;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    const uint32_t members = s_ex.members;
    const int wbeg = s_wbeg[warp], wend = s_wbeg[warp + 1];

    uint32_t cphase = 0;
    for (int pq = p0; pq < p1; pq += kMtTok) {
        const int nt = min(kMtTok, p1 - pq);
        const int npairs = (nt + 1) / 2;  // token pairs with a routed token (the second is skipped if empty)
        // ---- the c rows of this group's tokens (one bulk copy each; the first
        // group's went out before the staging) ----
        if (pq != p0) {
            __syncthreads();  // the previous group's c rows and partial sums are no longer read
            if (warp == 0) {
                const int pr = lane < nt ? P.rw.pairs[pq + lane] : -1;
                mt_issue_group(P, pr, nt, members, lane, s_pair, s_zp, s_c, &s_cbar);
            }
        }
        if (tid == 0 && !mt_mbar_wait(&s_cbar, cphase)) s_fail = 1;
        cphase ^= 1u;
        if (pq == p0) asm volatile("cp.async.wait_all;" ::: "memory");  // this thread's pieces of the planes
        __syncthreads();
        if (s_fail) {
            if (tid == 0 && P.status) atomicOr(P.status, BITSMOE_ST_TIMEOUT);
            return;
        }

        // acc[tile][pair]: this warp's partial sums for its rows of every tile
        float2 acc[kMtMaxTiles][kMtPairs];
#pragma unroll
        for (int t = 0; t < kMtMaxTiles; t++)
#pragma unroll
            for (int q = 0; q < kMtPairs; q++) acc[t][q] = make_float2(0.0f, 0.0f);

        // ---- this warp's member words, in group order: its own tables, then every
        // plane word of the member word for every tile of the CTA ----
        int g = 1, wg0 = 0;  // group of the current word, and its first word index
        for (int wi = wbeg; wi < wend; wi++) {
            while (g < kNumGroups - 1 && wi >= wg0 + (int)s_ex.W[g]) {
                wg0 += (int)s_ex.W[g];
                g++;
            }
            const int b = group_width(g), w = wi - wg0;
            const uint32_t W = s_ex.W[g];
            // this word's c values of token 0; token u's are members floats further on.  A
            // table's four members are one 16-byte load per token, shared by the 16 lanes
            // that build the table (a broadcast): no shuffles
            const float* cw = s_c + s_ex.c_off[g] + 32u * (uint32_t)w;
            __syncwarp();  // the previous word's lookups are done with the tables
            if (nt == 1) {
                // one token: float tables (8 x 16 entries, 512 B), one 4-byte lookup per
                // nibble -- half the shared-memory traffic of a token pair
                float* tab1 = reinterpret_cast<float*>(my_tab);
                const int e1 = lane & 15;
#pragma unroll
                for (int qq = 0; qq < 4; qq++) {
                    const int tb = (lane >> 4) + 2 * qq;
                    const float4 xv = *reinterpret_cast<const float4*>(cw + 4 * tb);
                    tab1[tb * 16 + e1] = ((e1 & 1 ? xv.x : 0.0f) + (e1 & 2 ? xv.y : 0.0f)) +
                                         ((e1 & 4 ? xv.z : 0.0f) + (e1 & 8 ? xv.w : 0.0f));
                }
                __syncwarp();
                const uint32_t* stg1 = s_stage + s_ex.stage_off[g] + (uint32_t)w * (uint32_t)ntl * 32u + (uint32_t)lane;
                for (int j = 0; j < b; j++) {
                    const float wt = (float)(1u << j);
                    const uint32_t* sj = stg1 + (uint32_t)j * W * (uint32_t)ntl * 32u;
#pragma unroll
                    for (int t = 0; t < kMtMaxTiles; t++) {
                        if (t >= ntl) break;
                        const uint32_t word = sj[t * 32];
                        // entry offsets (nibble x 4 bytes): even nibbles in the bytes of lo, odd in hi
                        const uint32_t lo = (word << 2) & 0x3C3C3C3Cu, hi = (word >> 2) & 0x3C3C3C3Cu;
                        const float sum =
                            ((mt_lds1<0>(__byte_perm(lo, my_tab_s, 0x7650u)) + mt_lds1<64>(__byte_perm(hi, my_tab_s, 0x7650u))) +
                             (mt_lds1<128>(__byte_perm(lo, my_tab_s, 0x7651u)) + mt_lds1<192>(__byte_perm(hi, my_tab_s, 0x7651u)))) +
                            ((mt_lds1<256>(__byte_perm(lo, my_tab_s, 0x7652u)) + mt_lds1<320>(__byte_perm(hi, my_tab_s, 0x7652u))) +
                             (mt_lds1<384>(__byte_perm(lo, my_tab_s, 0x7653u)) + mt_lds1<448>(__byte_perm(hi, my_tab_s, 0x7653u))));
                        acc[t][0].x = fmaf(sum, wt, acc[t][0].x);
                    }
                }
                continue;
            }
            // entry en of table tb of pair pr = the sums of c over the set bits of en
            // (members 4 tb .. 4 tb + 3) for tokens 2 pr and 2 pr + 1; a token past the
            // group's last (its c row holds an earlier group's values) counts as 0
            const int en = lane & 15;
#pragma unroll
            for (int pr = 0; pr < kMtPairs; pr++) {
                if (pr >= npairs) break;
                const bool has_y = 2 * pr + 1 < nt;
                const float* cx = cw + (size_t)(2 * pr) * members;
#pragma unroll
                for (int qq = 0; qq < 4; qq++) {
                    const int tb = (lane >> 4) + 2 * qq;
                    const float4 xv = *reinterpret_cast<const float4*>(cx + 4 * tb);
                    float4 yv = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    if (has_y) yv = *reinterpret_cast<const float4*>(cx + members + 4 * tb);
                    float2 v;
                    v.x = ((en & 1 ? xv.x : 0.0f) + (en & 2 ? xv.y : 0.0f)) + ((en & 4 ? xv.z : 0.0f) + (en & 8 ? xv.w : 0.0f));
                    v.y = ((en & 1 ? yv.x : 0.0f) + (en & 2 ? yv.y : 0.0f)) + ((en & 4 ? yv.z : 0.0f) + (en & 8 ? yv.w : 0.0f));
                    my_tab[(pr * 8 + tb) * 16 + en] = v;
                }
            }
            __syncwarp();  // the tables are written
            const uint32_t* stg = s_stage + s_ex.stage_off[g] + (uint32_t)w * (uint32_t)ntl * 32u + (uint32_t)lane;
            for (int j = 0; j < b; j++) {
                const float wt = (float)(1u << j);
                const uint32_t* sj = stg + (uint32_t)j * W * (uint32_t)ntl * 32u;
#pragma unroll
                for (int t = 0; t < kMtMaxTiles; t++) {
                    if (t >= ntl) break;
                    const uint32_t word = sj[t * 32];
                    // entry offsets (nibble x 8 bytes): even nibbles in the bytes of lo, odd in hi
                    const uint32_t lo = (word << 3) & 0x78787878u, hi = (word >> 1) & 0x78787878u;
                    const uint32_t a0 = __byte_perm(lo, my_tab_s, 0x7650u), a1 = __byte_perm(hi, my_tab_s, 0x7650u);
                    const uint32_t a2 = __byte_perm(lo, my_tab_s, 0x7651u), a3 = __byte_perm(hi, my_tab_s, 0x7651u);
                    const uint32_t a4 = __byte_perm(lo, my_tab_s, 0x7652u), a5 = __byte_perm(hi, my_tab_s, 0x7652u);
                    const uint32_t a6 = __byte_perm(lo, my_tab_s, 0x7653u), a7 = __byte_perm(hi, my_tab_s, 0x7653u);
                    {
                        const float2 s = f2add(f2add(f2add(mt_lds2<0>(a0), mt_lds2<128>(a1)),
                                                     f2add(mt_lds2<256>(a2), mt_lds2<384>(a3))),
                                               f2add(f2add(mt_lds2<512>(a4), mt_lds2<640>(a5)),
                                                     f2add(mt_lds2<768>(a6), mt_lds2<896>(a7))));
                        acc[t][0].x = fmaf(s.x, wt, acc[t][0].x);
                        acc[t][0].y = fmaf(s.y, wt, acc[t][0].y);
                    }
                    if (npairs > 1) {
                        const float2 s = f2add(f2add(f2add(mt_lds2<1024>(a0), mt_lds2<1152>(a1)),
                                                     f2add(mt_lds2<1280>(a2), mt_lds2<1408>(a3))),
                                               f2add(f2add(mt_lds2<1536>(a4), mt_lds2<1664>(a5)),
                                                     f2add(mt_lds2<1792>(a6), mt_lds2<1920>(a7))));
                        acc[t][1].x = fmaf(s.x, wt, acc[t][1].x);
                        acc[t][1].y = fmaf(s.y, wt, acc[t][1].y);
                    }
                }
            }
        }
        // fp16 group: (a_k z_{t,k}) w16_{k,i}, rows read in place; member m to warp m % warps
        if (s_ex.n[0] > 0) {
            const uint32_t np = s_ex.np[0];
            const uint16_t* w16 = reinterpret_cast<const uint16_t*>(P.blob + s_ex.gbase[0] + 6ull * np);
            const float* c16 = s_c + s_ex.c_off[0];
            for (uint32_t mm = warp; mm < s_ex.n[0]; mm += kMtWarps) {
                const float cz0 = c16[mm], cz1 = c16[members + mm], cz2 = c16[2 * members + mm],
                            cz3 = c16[3 * members + mm];
#pragma unroll
                for (int t = 0; t < kMtMaxTiles; t++) {
                    if (t >= ntl) break;
                    const int row = (tile0 + t) * 32 + lane;
                    const float wv = __half2float(__ushort_as_half(w16[(size_t)mm * P.d_pad + row]));
                    acc[t][0].x = fmaf(cz0, wv, acc[t][0].x);
                    acc[t][0].y = fmaf(cz1, wv, acc[t][0].y);
                    acc[t][1].x = fmaf(cz2, wv, acc[t][1].x);
                    acc[t][1].y = fmaf(cz3, wv, acc[t][1].y);
                }
            }
        }
        // ---- the warps' partial sums, added in warp order; warp t writes tile t ----
        __syncthreads();  // every warp is done with its tables: s_part reuses them
#pragma unroll
        for (int t = 0; t < kMtMaxTiles; t++) {
            if (t >= ntl) break;
            float* pp = s_part + (((size_t)warp * kMtMaxTiles + t) * 32 + lane) * kMtTok;
            pp[0] = acc[t][0].x;
            pp[1] = acc[t][0].y;
            pp[2] = acc[t][1].x;
            pp[3] = acc[t][1].y;
        }
        __syncthreads();
        for (int t = warp; t < ntl; t += kMtWarps) {
            const int row = (tile0 + t) * 32 + lane;
            if (row >= P.d_out) continue;
            float y[kMtTok];
#pragma unroll
            for (int u = 0; u < kMtTok; u++) y[u] = -s_zp[u];
            for (int v = 0; v < kMtWarps; v++) {
                const float* pp = s_part + (((size_t)v * kMtMaxTiles + t) * 32 + lane) * kMtTok;
#pragma unroll
                for (int u = 0; u < kMtTok; u++) y[u] += pp[u];
            }
#pragma unroll
            for (int u = 0; u < kMtTok; u++)
                if (u < nt && in_bounds(s_pair[u], (uint64_t)P.n_pairs, P.status))
                    P.Ye[(size_t)s_pair[u] * P.d_out + row] = y[u];
        }
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

// Floats per c row: every expert's padded members, rounded to 8 (32-byte rows).
uint32_t cvals_ldc(const bitsmoe_plan* p) { return (uint32_t)roundup(p->max_members_padded, 8); }

int launch_expert_mt(const bitsmoe_plan* p, const void* blob, const float* Z, const int32_t* ids, int T,
                     const RouteWS& rw, float* Ye, int32_t* status, cudaStream_t s) {
    // the current device's shared-memory limit, looked up on every call (a host-side
    // query; a process may drive devices of different limits)
    int max_smem = 0;
    {
        int dev;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return set_cuda_error(e);
    }
    if (rw.ldc < cvals_ldc(p)) return BITSMOE_EINVAL;
    const int npairs = T * p->dims.top_k;
    k_cvals<<<(unsigned)npairs, kCvThreads, 0, s>>>((const uint8_t*)blob, Z, ids, p->dims.top_k, p->dims.n_experts,
                                                    p->dims.rank, rw);
    int rc = check_launch();
    if (rc) return rc;

    MtParams P{};
    P.blob = (const uint8_t*)blob;
    P.blob_bytes = p->blob_bytes;
    P.n_pairs = npairs;
    P.rw = rw;
    P.Ye = Ye;
    P.status = status;
    P.K = p->dims.top_k;
    P.d_out = p->dims.d_out;
    P.d_pad = (int)p->d_pad;
    P.n_tiles = (int)(p->d_pad / 32);
    // per-expert maximum of the words of one tile over the bit-plane groups
    uint64_t tile_words = 0;
    for (int e = 0; e < p->dims.n_experts; e++) {
        const uint32_t* c = p->counts + 8 * (size_t)e;
        uint64_t tw = 0;
        for (int g = 0; g < kNumGroups; g++) {
            const int b = group_width(g);
            if (b != 16) tw += (uint64_t)b * (group_members_padded(b, c[g]) / 32) * 32;
        }
        tile_words = std::max(tile_words, tw);
    }
    // c rows of kMtTok tokens, and each warp's tables (2 KB, + 1024 for their
    // alignment), which the warps' partial sums reuse at the end
    static_assert(kMtWarps * kMtMaxTiles * 32 * kMtTok * 4 <= kMtWarps * 2048, "partial sums fit the tables");
    const uint64_t fixed = roundup(4ull * kMtTok * p->max_members_padded, 128) + kMtWarps * 2048ull + 1024 + 128;
    const uint64_t budget = (uint64_t)max_smem - 1024;  // static shared memory of the kernel
    // the most tiles per CTA that still lets two CTAs share an SM (one stages while
    // the other computes); else the most that fit one CTA per SM
    const uint64_t half = (uint64_t)max_smem / 2 - 1024;
    int tpc = kMtMaxTiles;
    while (tpc > 1 && fixed + 4 * tile_words * tpc > half) tpc /= 2;
    if (fixed + 4 * tile_words * tpc > half) {
        tpc = kMtMaxTiles;
        while (tpc > 1 && fixed + 4 * tile_words * tpc > budget) tpc /= 2;
    }
    if (fixed + 4 * tile_words * tpc > budget) return BITSMOE_ESIZE;  // one tile does not fit
    P.tiles_per_cta = tpc;
    P.sm_stage = 0;
    P.sm_c = (uint32_t)roundup(4ull * tile_words * tpc, 128);
    P.sm_tab = P.sm_c + (uint32_t)roundup(4ull * kMtTok * p->max_members_padded, 128);
    P.stage_words = (uint32_t)(tile_words * tpc);
    P.c_floats = (uint32_t)(kMtTok * p->max_members_padded);
    const size_t smem = P.sm_tab + kMtWarps * 2048 + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_expert_mt, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return set_cuda_error(e);
    const int slots = (int)std::min<int64_t>((int64_t)p->dims.n_experts, (int64_t)npairs);
    dim3 grid((unsigned)slots, (unsigned)((P.n_tiles + tpc - 1) / tpc));
    k_expert_mt<<<grid, kMtThreads, smem, s>>>(P);
    return check_launch();
}

}  // namespace bitsmoe
