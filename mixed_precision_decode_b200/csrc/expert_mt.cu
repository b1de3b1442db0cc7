// expert_mt.cu -- routed expert forward for any number of tokens: the
// width-grouped bit planes of one expert, evaluated bit-serially for every
// token routed to it (BitsMoE study-note page, Methodology: W_e x =
// P_e A_e (Phi^T x); Execution: bit planes grouped by width):
//   y_{t,i} = sum_b sum_j 2^j sum_{k in G_b} c_{k,t} bit_{k,j,i}
//             - sum_b (2^b - 1)/2 sum_{k in G_b} c_{k,t}
//             + sum_{k in G_16} a_k z_{t,k} w16_{k,i},        c_{k,t} = a_k s_k z_{t,k}.
//
// Design: one CTA per (routed expert, range of 32-row tiles).  The CTA stages
// its tiles' planes and the expert's per-component metadata in shared memory
// with a few TMA bulk copies (a run of tiles of one group is contiguous), then
// loops over the expert's tokens in groups of four.  Per group it forms c for
// every member and token, and per chunk of 128 members it builds 16-entry
// subset-sum tables whose entries are token PAIRS (float2): one conflict-free
// 8-byte shared load answers a 4-member nibble for two tokens, so the
// bit-serial sum costs one byte-permute and two loads per nibble for four
// tokens.  A warp owns one 32-row tile (a lane per row); when a CTA stages
// fewer than 8 tiles, several warps share a tile and split its plane words.
#include <algorithm>

#include "common.cuh"

namespace bitsmoe {

constexpr int kMtThreads = 256;
constexpr int kMtWarps = kMtThreads / 32;
constexpr int kMtTok = 4;           // tokens per group
constexpr int kMtPairs = kMtTok / 2;
constexpr int kMtCW = 4;            // 32-member words per chunk
constexpr long long kMtWaitNs = 2000000000LL;

struct MtParams {
    const uint8_t* blob;
    const float* Z;
    RouteWS rw;
    float* Ye;
    int32_t* status;
    int r, K, d_out, d_pad, n_tiles;
    int tiles_per_cta;  // 1, 2, 4 or 8 (warps per tile = 8 / tiles_per_cta)
    uint32_t stage_words, meta_bytes, c_floats;
    uint32_t sm_stage, sm_meta, sm_c, sm_tab, sm_misc;
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
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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

// Per-expert shape of the staged data.
struct MtExpert {
    uint32_t n[kNumGroups], np[kNumGroups], W[kNumGroups];
    uint32_t stage_off[kNumGroups];  // word offset of the group's tiles in the staging buffer
    uint32_t meta_off[kNumGroups];   // byte offset of the group's metadata in the staging buffer
    uint32_t c_off[kNumGroups];      // member offset of the group in the c buffer (bit-plane groups)
    uint64_t gbase[kNumGroups];      // byte offset of the group in the blob
    uint32_t members;                // padded bit-plane members
};

__global__ void __launch_bounds__(kMtThreads) k_expert_mt(const MtParams P) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint64_t s_bar;
    __shared__ MtExpert s_ex;
    __shared__ int s_tok[kMtTok], s_pair[kMtTok], s_fail;
    __shared__ float s_zpw[kMtWarps][kMtTok], s_zpt[kMtTok];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int slot = blockIdx.x;
    if (slot >= *P.rw.nactive) return;
    const int e = P.rw.active[slot];
    const int p0 = P.rw.start[e], p1 = P.rw.start[e + 1];
    const int tile0 = blockIdx.y * P.tiles_per_cta;
    const int ntl = min(P.tiles_per_cta, P.n_tiles - tile0);
    if (ntl <= 0) return;
    const int wpt = kMtWarps / P.tiles_per_cta;  // warps per tile
    const int my_tile = warp / wpt, part = warp % wpt;
    const int row = (tile0 + my_tile) * 32 + lane;
    const bool tile_ok = my_tile < ntl;

    uint32_t* s_stage = reinterpret_cast<uint32_t*>(smem + P.sm_stage);
    uint8_t* s_meta = smem + P.sm_meta;
    float* s_c = reinterpret_cast<float*>(smem + P.sm_c);  // [member][kMtTok]
    // token-pair tables: 1024-byte aligned blocks of (word, pair) -> 8 nibble tables x 16 float2
    const uint32_t tab_raw = mt_smem_u32(smem + P.sm_tab);
    const uint32_t tab_s = (tab_raw + 1023u) & ~1023u;
    float2* s_tab = reinterpret_cast<float2*>(smem + P.sm_tab + (tab_s - tab_raw));
    float* s_red = reinterpret_cast<float*>(s_tab);  // reused after the last chunk: [warp][32][kMtTok]

    // ---- stage the expert's metadata and this CTA's rows of every plane word ----
    if (warp == 0) {
      if (lane == 0) {
        const DirEntry d = read_dir(P.blob, e);
        uint32_t so = 0, mo = 0, co = 0;
        for (int g = 0; g < kNumGroups; g++) {
            const int b = group_width(g);
            s_ex.n[g] = d.count[g];
            s_ex.np[g] = (uint32_t)group_members_padded(b, d.count[g]);
            s_ex.W[g] = b == 16 ? 0 : s_ex.np[g] / 32;
            s_ex.stage_off[g] = so;
            s_ex.meta_off[g] = mo;
            s_ex.c_off[g] = co;
            s_ex.gbase[g] = d.base + d.goff[g];
            if (b != 16) {
                so += (uint32_t)ntl * b * s_ex.W[g] * 32;
                co += s_ex.np[g];
            }
            mo += (b == 16 ? 6u : 8u) * s_ex.np[g];
        }
        s_ex.members = co;
        s_fail = 0;
        mt_mbar_init(&s_bar);
        mt_expect_tx(&s_bar, 4 * so + mo);
        for (int g = 0; g < kNumGroups; g++) {
            if (s_ex.n[g] == 0) continue;
            const int b = group_width(g);
            mt_bulk(s_meta + s_ex.meta_off[g], P.blob + s_ex.gbase[g], (b == 16 ? 6u : 8u) * s_ex.np[g], &s_bar);
        }
      }
      __syncwarp();
      // plane word q of group g: rows [32 tile0, 32 (tile0 + ntl)) are contiguous in the
      // blob ([b][W][d_pad], rows fastest) and staged as [b][W][32 ntl]
      const uint64_t d_pad = 32ull * P.n_tiles;
      int g = 1, qg = 0;  // group of plane word q, and its first word
      for (int q = lane;; q += 32) {
          while (g < kNumGroups && q >= qg + group_width(g) * (int)s_ex.W[g]) {
              qg += group_width(g) * (int)s_ex.W[g];
              g++;
          }
          if (g >= kNumGroups) break;
          const uint8_t* planes = P.blob + s_ex.gbase[g] + 8ull * s_ex.np[g];
          mt_bulk(s_stage + s_ex.stage_off[g] + (uint32_t)(q - qg) * 32u * ntl,
                  planes + 4ull * ((uint64_t)(q - qg) * d_pad + 32ull * tile0), 128u * ntl, &s_bar);
      }
      if (lane == 0 && !mt_mbar_wait(&s_bar, 0)) {
          s_fail = 1;
          if (P.status) atomicOr(P.status, BITSMOE_ST_TIMEOUT);
      }
    }
    __syncthreads();
    if (s_fail) return;

    const int myt = tid % kMtTok;  // token whose c values this thread forms
    for (int pq = p0; pq < p1; pq += kMtTok) {
        const int nt = min(kMtTok, p1 - pq);
        __syncthreads();  // the previous group's outputs are written
        if (tid < kMtTok) {
            const int pr = tid < nt ? P.rw.pairs[pq + tid] : -1;
            s_pair[tid] = pr;
            s_tok[tid] = pr >= 0 ? pr / P.K : -1;
        }
        __syncthreads();
        // c_{k,t} = a_k s_k z_{t,k} of every bit-plane member, and the zero-point partials
        {
            const int tok = s_tok[myt];
            const float* zt = P.Z + (size_t)(tok < 0 ? 0 : tok) * P.r;
            float zp = 0.0f;
            for (int g = 1; g < kNumGroups; g++) {
                const uint32_t np = s_ex.np[g], n = s_ex.n[g];
                if (np == 0) continue;
                const uint8_t* gm = s_meta + s_ex.meta_off[g];
                const uint16_t* idx = reinterpret_cast<const uint16_t*>(gm);
                const uint16_t* scl = reinterpret_cast<const uint16_t*>(gm + 2 * np);
                const float* amp = reinterpret_cast<const float*>(gm + 4 * np);
                const float hr = 0.5f * (float)((1 << group_width(g)) - 1);
                float* cg = s_c + (size_t)s_ex.c_off[g] * kMtTok;
                // four values per pass: every load of a pass is issued before its stores
                for (uint32_t v0 = tid; v0 < np * kMtTok; v0 += 4 * kMtThreads) {
                    float c[4];
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        const uint32_t v = v0 + u * kMtThreads, m = v / kMtTok;
                        c[u] = (v < np * kMtTok && m < n && tok >= 0)
                                   ? amp[m] * __half2float(__ushort_as_half(scl[m])) * __ldg(zt + idx[m])
                                   : 0.0f;
                    }
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        const uint32_t v = v0 + u * kMtThreads;
                        if (v < np * kMtTok) cg[v] = c[u];
                        zp += hr * c[u];
                    }
                }
            }
            // lanes with equal lane % kMtTok hold the same token
            for (int o = kMtTok; o < 32; o <<= 1) zp += __shfl_xor_sync(0xffffffffu, zp, o);
            if (lane < kMtTok) s_zpw[warp][lane] = zp;
        }
        __syncthreads();
        if (tid < kMtTok) {
            float s = 0.0f;
            for (int w = 0; w < kMtWarps; w++) s += s_zpw[w][tid];
            s_zpt[tid] = s;
        }
        float2 acc[kMtPairs];
#pragma unroll
        for (int q = 0; q < kMtPairs; q++) acc[q] = make_float2(0.0f, 0.0f);

        for (int g = 1; g < kNumGroups; g++) {
            const int b = group_width(g);
            const uint32_t W = s_ex.W[g];
            if (W == 0) continue;
            const float* cg = s_c + (size_t)s_ex.c_off[g] * kMtTok;
            const uint32_t* stg = s_stage + s_ex.stage_off[g];
            for (uint32_t w0 = 0; w0 < W; w0 += kMtCW) {
                const int cw = (int)min((uint32_t)kMtCW, W - w0);
                __syncthreads();  // the previous chunk's tables are no longer read
                // entry x = ((wi * kMtPairs + pair) * 8 + n) * 16 + e: sum of c over the set bits of e
                for (int x = tid; x < cw * kMtPairs * 128; x += kMtThreads) {
                    const int en = x & 15, n = (x >> 4) & 7, wp = x >> 7;
                    const int pair = wp % kMtPairs, wi = wp / kMtPairs;
                    const float* cm = cg + (size_t)(32 * (w0 + wi) + 4 * n) * kMtTok + 2 * pair;
                    float2 v = make_float2(0.0f, 0.0f);
#pragma unroll
                    for (int bit = 0; bit < 4; bit++)
                        if (en & (1 << bit)) v = f2add(v, *reinterpret_cast<const float2*>(cm + bit * kMtTok));
                    s_tab[x] = v;
                }
                __syncthreads();
                if (!tile_ok) continue;
                for (int q = part; q < b * cw; q += wpt) {
                    const int j = q / cw, wi = q - j * cw;
                    const uint32_t word = stg[(((uint32_t)j * W + w0 + wi) * ntl + my_tile) * 32 + lane];
                    // entry offsets (nibble x 8 bytes): even nibbles in the bytes of lo, odd in hi
                    const uint32_t lo = (word << 3) & 0x78787878u, hi = (word >> 1) & 0x78787878u;
                    const uint32_t base = tab_s + 2048u * (uint32_t)wi;  // (wi, pair 0); pair 1 at +1024
                    const uint32_t a0 = __byte_perm(lo, base, 0x7650u), a1 = __byte_perm(hi, base, 0x7650u);
                    const uint32_t a2 = __byte_perm(lo, base, 0x7651u), a3 = __byte_perm(hi, base, 0x7651u);
                    const uint32_t a4 = __byte_perm(lo, base, 0x7652u), a5 = __byte_perm(hi, base, 0x7652u);
                    const uint32_t a6 = __byte_perm(lo, base, 0x7653u), a7 = __byte_perm(hi, base, 0x7653u);
                    const float wt = (float)(1u << j);
                    {
                        const float2 s = f2add(f2add(f2add(mt_lds2<0>(a0), mt_lds2<128>(a1)),
                                                     f2add(mt_lds2<256>(a2), mt_lds2<384>(a3))),
                                               f2add(f2add(mt_lds2<512>(a4), mt_lds2<640>(a5)),
                                                     f2add(mt_lds2<768>(a6), mt_lds2<896>(a7))));
                        acc[0].x = fmaf(s.x, wt, acc[0].x);
                        acc[0].y = fmaf(s.y, wt, acc[0].y);
                    }
                    {
                        const float2 s = f2add(f2add(f2add(mt_lds2<1024>(a0), mt_lds2<1152>(a1)),
                                                     f2add(mt_lds2<1280>(a2), mt_lds2<1408>(a3))),
                                               f2add(f2add(mt_lds2<1536>(a4), mt_lds2<1664>(a5)),
                                                     f2add(mt_lds2<1792>(a6), mt_lds2<1920>(a7))));
                        acc[1].x = fmaf(s.x, wt, acc[1].x);
                        acc[1].y = fmaf(s.y, wt, acc[1].y);
                    }
                }
            }
        }
        // fp16 group: a_k z_{t,k} w16_{k,i}
        if (s_ex.n[0] > 0 && tile_ok && row < P.d_out) {
            const uint32_t np = s_ex.np[0];
            const uint8_t* gm = s_meta + s_ex.meta_off[0];
            const uint16_t* idx = reinterpret_cast<const uint16_t*>(gm);
            const float* amp = reinterpret_cast<const float*>(gm + 2 * np);
            const uint16_t* w16 = reinterpret_cast<const uint16_t*>(P.blob + s_ex.gbase[0] + 6ull * np);
            for (uint32_t m = part; m < s_ex.n[0]; m += wpt) {
                const float wv = __half2float(__ushort_as_half(w16[(size_t)m * P.d_pad + row]));
                float cz[kMtTok];
#pragma unroll
                for (int t = 0; t < kMtTok; t++)
                    cz[t] = s_tok[t] >= 0 ? amp[m] * __ldg(P.Z + (size_t)s_tok[t] * P.r + idx[m]) : 0.0f;
                acc[0].x = fmaf(cz[0], wv, acc[0].x);
                acc[0].y = fmaf(cz[1], wv, acc[0].y);
                acc[1].x = fmaf(cz[2], wv, acc[1].x);
                acc[1].y = fmaf(cz[3], wv, acc[1].y);
            }
        }
        // warps sharing a tile add their partial sums; the first writes the rows
        __syncthreads();  // tables are no longer read: s_red reuses them
        float* red = s_red + ((size_t)warp * 32 + lane) * kMtTok;
        red[0] = acc[0].x;
        red[1] = acc[0].y;
        red[2] = acc[1].x;
        red[3] = acc[1].y;
        __syncthreads();
        if (part == 0 && tile_ok && row < P.d_out) {
            float y[kMtTok];
#pragma unroll
            for (int t = 0; t < kMtTok; t++) y[t] = -s_zpt[t];
            for (int w = warp; w < warp + wpt; w++) {
                const float* rr = s_red + ((size_t)w * 32 + lane) * kMtTok;
#pragma unroll
                for (int t = 0; t < kMtTok; t++) y[t] += rr[t];
            }
#pragma unroll
            for (int t = 0; t < kMtTok; t++)
                if (t < nt) P.Ye[(size_t)s_pair[t] * P.d_out + row] = y[t];
        }
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int g_mt_max_smem = 0;

int launch_expert_mt(const bitsmoe_plan* p, const void* blob, const float* Z, int T, const RouteWS& rw, float* Ye,
                     int32_t* status, cudaStream_t s) {
    if (g_mt_max_smem == 0) {
        int dev;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&g_mt_max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return set_cuda_error(e);
    }
    MtParams P{};
    P.blob = (const uint8_t*)blob;
    P.Z = Z;
    P.rw = rw;
    P.Ye = Ye;
    P.status = status;
    P.r = p->dims.rank;
    P.K = p->dims.top_k;
    P.d_out = p->dims.d_out;
    P.d_pad = (int)p->d_pad;
    P.n_tiles = (int)(p->d_pad / 32);
    // per-expert maxima: words of one tile over the bit-plane groups, metadata bytes, members
    uint64_t tile_words = 0, meta = 0, members = 0;
    for (int e = 0; e < p->dims.n_experts; e++) {
        const uint32_t* c = p->counts + 8 * (size_t)e;
        uint64_t tw = 0, mb = 0, mm = 0;
        for (int g = 0; g < kNumGroups; g++) {
            const int b = group_width(g);
            const uint64_t np = group_members_padded(b, c[g]);
            mb += (b == 16 ? 6 : 8) * np;
            if (b != 16) {
                tw += (uint64_t)b * (np / 32) * 32;
                mm += np;
            }
        }
        tile_words = std::max(tile_words, tw);
        meta = std::max(meta, mb);
        members = std::max(members, mm);
    }
    const uint64_t fixed = roundup(meta, 128) + roundup(members * kMtTok * 4, 128) + 8192 + 1024 + 128;
    const uint64_t budget = (uint64_t)g_mt_max_smem - 1024;  // static shared memory of the kernel
    // the most tiles per CTA that still lets two CTAs share an SM (more warps hide the
    // shared-memory latency of the lookups); else the most that fit one CTA per SM
    const uint64_t half = (uint64_t)g_mt_max_smem / 2 - 1024;
    int tpc = 8;
    while (tpc > 1 && fixed + 4 * tile_words * tpc > half) tpc /= 2;
    if (fixed + 4 * tile_words * tpc > half) {
        tpc = 8;
        while (tpc > 1 && fixed + 4 * tile_words * tpc > budget) tpc /= 2;
    }
    if (fixed + 4 * tile_words * tpc > budget) return BITSMOE_ESIZE;  // one tile does not fit
    P.tiles_per_cta = tpc;
    P.stage_words = (uint32_t)(tile_words * tpc);
    P.meta_bytes = (uint32_t)roundup(meta, 128);
    P.c_floats = (uint32_t)(members * kMtTok);
    P.sm_stage = 0;
    P.sm_meta = (uint32_t)roundup(4ull * P.stage_words, 128);
    P.sm_c = P.sm_meta + P.meta_bytes;
    P.sm_tab = (uint32_t)(P.sm_c + roundup(4ull * P.c_floats, 128));
    const size_t smem = P.sm_tab + 8192 + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_expert_mt, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return set_cuda_error(e);
    const int slots = (int)std::min<int64_t>((int64_t)p->dims.n_experts, (int64_t)T * P.K);
    dim3 grid((unsigned)slots, (unsigned)((P.n_tiles + tpc - 1) / tpc));
    k_expert_mt<<<grid, kMtThreads, smem, s>>>(P);
    return check_launch();
}

}  // namespace bitsmoe
