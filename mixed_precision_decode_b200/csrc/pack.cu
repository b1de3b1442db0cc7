// pack.cu -- per-component fp16 scales, width-grouped bit-plane packing and
// the test-support unpack (BitsMoE study-note page, sections "Usage" and
// "Execution": widths {0,1,2,3,4,6,8,16}; equal widths grouped, packed by
// bit plane).  Offline work: one streaming pass over the fp32 components.
#include "common.cuh"

namespace bitsmoe {

// ---------------------------------------------------------------------------
// scales: one warp per component
// ---------------------------------------------------------------------------
__global__ void k_compute_scales(const float* __restrict__ comps, const uint8_t* __restrict__ widths,
                                 uint16_t* __restrict__ scales, int32_t* status, uint64_t n_comp, int d_out) {
    uint64_t c = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int lane = threadIdx.x & 31;
    if (c >= n_comp) return;
    int b = widths[c];
    if (b == 0 || b == 16 || !width_ok(b)) {
        if (lane == 0) {
            scales[c] = 0;
            if (!width_ok(b) && status) atomicOr(status, BITSMOE_ST_PLANMISMATCH);
        }
        return;
    }
    const float* p = comps + c * (uint64_t)d_out;
    float m = 0.0f;
    bool bad = false;
    for (int i = lane; i < d_out; i += 32) {
        float v = p[i];
        bad |= !isfinite(v);
        m = fmaxf(m, fabsf(v));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
        if (bad) {
            scales[c] = 0;
            if (status) atomicOr(status, BITSMOE_ST_NONFINITE);
        } else {
            float two_m = __fmul_rn(2.0f, m);
            float s32 = __fdiv_rn(two_m, (float)((1 << b) - 1));
            scales[c] = __half_as_ushort(__float2half_rn(s32));
        }
    }
}

// ---------------------------------------------------------------------------
// pack, step 1: member lists, scales and amplitudes (one CTA per expert)
// ---------------------------------------------------------------------------
constexpr int kIndexThreads = 256;

__global__ void __launch_bounds__(kIndexThreads) k_pack_index(const uint8_t* __restrict__ widths,
                                                              const uint16_t* __restrict__ scales,
                                                              const float* __restrict__ amps, uint8_t* blob, int r,
                                                              int32_t* status) {
    extern __shared__ uint8_t s_w[];  // r widths of this expert
    __shared__ uint32_t s_cnt[kNumGroups][kIndexThreads];
    __shared__ uint32_t s_tot[kNumGroups];
    __shared__ int s_bad;
    const int e = blockIdx.x, tid = threadIdx.x;
    const uint8_t* wrow = widths + (uint64_t)e * r;
    for (int k = tid; k < r; k += blockDim.x) s_w[k] = wrow[k];
    if (tid == 0) s_bad = 0;
    __syncthreads();
    // contiguous chunk of k per thread keeps ascending-k order inside each group
    const int chunk = (r + blockDim.x - 1) / blockDim.x;
    const int k0 = min(r, tid * chunk), k1 = min(r, k0 + chunk);
    uint32_t loc[kNumGroups] = {0, 0, 0, 0, 0, 0, 0};
    for (int k = k0; k < k1; k++) {
        int g = group_of_width(s_w[k]);
        if (g >= 0) loc[g]++;
        else if (s_w[k] != 0) s_bad = 1;
    }
#pragma unroll
    for (int g = 0; g < kNumGroups; g++) s_cnt[g][tid] = loc[g];
    __syncthreads();
    if (tid < kNumGroups) {  // exclusive scan, one group per thread
        uint32_t run = 0;
        for (int t = 0; t < (int)blockDim.x; t++) {
            uint32_t v = s_cnt[tid][t];
            s_cnt[tid][t] = run;
            run += v;
        }
        s_tot[tid] = run;
    }
    __syncthreads();
    const DirEntry d = read_dir(blob, e);
    if (tid == 0) {
        bool mismatch = s_bad != 0;
        for (int g = 0; g < kNumGroups; g++) mismatch |= s_tot[g] != d.count[g];
        s_bad = mismatch ? 1 : 0;
        if (mismatch && status) atomicOr(status, BITSMOE_ST_PLANMISMATCH);
    }
    __syncthreads();
    if (s_bad) return;  // leave the expert zero; the status word says why
    uint32_t slot[kNumGroups];
#pragma unroll
    for (int g = 0; g < kNumGroups; g++) slot[g] = s_cnt[g][tid];
    for (int k = k0; k < k1; k++) {
        int g = group_of_width(s_w[k]);
        if (g < 0) continue;
        uint32_t m = slot[g]++;
        uint8_t* G = blob + d.base + d.goff[g];
        uint64_t np = group_members_padded(group_width(g), d.count[g]);
        reinterpret_cast<uint16_t*>(G)[m] = (uint16_t)k;
        float a = amps[(uint64_t)e * r + k];
        if (g == 0) {
            reinterpret_cast<float*>(G + 2 * np)[m] = a;
        } else {
            reinterpret_cast<uint16_t*>(G + 2 * np)[m] = scales[(uint64_t)e * r + k];
            reinterpret_cast<float*>(G + 4 * np)[m] = a;
        }
    }
}

// Work items of one expert: its fp16 members one by one, then the 32-member
// words of the bit-plane groups in storage order.
struct Item {
    int g;       // group (0 = fp16)
    uint32_t w;  // member (fp16 group) or word index
};
__device__ inline bool item_of(const DirEntry& d, uint32_t it, Item& out) {
    if (it < d.count[0]) {
        out.g = 0;
        out.w = it;
        return true;
    }
    it -= d.count[0];
    for (int g = 1; g < kNumGroups; g++) {
        uint32_t W = (uint32_t)(group_members_padded(group_width(g), d.count[g]) / 32);
        if (it < W) {
            out.g = g;
            out.w = it;
            return true;
        }
        it -= W;
    }
    return false;
}

// ---------------------------------------------------------------------------
// pack, step 2: quantise and scatter bits (grid: expert x item x row blocks)
// ---------------------------------------------------------------------------
template <int B>
__device__ void pack_word(const float* __restrict__ comps_e, const uint16_t* idx, const uint16_t* scl, uint32_t n,
                          uint32_t w, uint32_t W, int d_out, uint32_t d_pad, uint32_t* planes, int& st) {
    __shared__ uint16_t s_k[32], s_s[32];
    __syncthreads();  // the previous item of this block may still read s_k / s_s
    if (threadIdx.x < 32) {
        uint32_t m = 32 * w + threadIdx.x;
        s_k[threadIdx.x] = m < n ? idx[m] : 0;
        s_s[threadIdx.x] = m < n ? scl[m] : 0;
    }
    __syncthreads();
    const uint32_t valid = min(32u, n - 32 * w);
    for (uint32_t i = blockIdx.z * blockDim.x + threadIdx.x; i < (uint32_t)d_out; i += gridDim.z * blockDim.x) {
        uint32_t word[B];
#pragma unroll
        for (int j = 0; j < B; j++) word[j] = 0;
        for (uint32_t m = 0; m < valid; m++) {
            float p = comps_e[(uint64_t)s_k[m] * d_out + i];
            uint32_t q = quantise(p, B, s_s[m], st);
#pragma unroll
            for (int j = 0; j < B; j++) word[j] |= ((q >> j) & 1u) << m;
        }
#pragma unroll
        for (int j = 0; j < B; j++) planes[plane_word(j, w, W, d_pad, i)] = word[j];
    }
}

__global__ void k_pack_planes(const float* __restrict__ comps, uint8_t* blob, int r, int d_out, uint32_t d_pad,
                              int32_t* status) {
    const int e = blockIdx.x;
    const DirEntry d = read_dir(blob, e);
    const float* comps_e = comps + (uint64_t)e * r * d_out;
    int st = 0;
    Item item;
    for (uint32_t it = blockIdx.y; item_of(d, it, item); it += gridDim.y) {
    if (item.g == 0) {
        HGroup h = hgroup(blob, d);
        uint32_t k = h.idx[item.w];
        uint16_t* w16 = const_cast<uint16_t*>(h.w16) + (uint64_t)item.w * d_pad;
        for (uint32_t i = blockIdx.z * blockDim.x + threadIdx.x; i < (uint32_t)d_out; i += gridDim.z * blockDim.x) {
            float p = comps_e[(uint64_t)k * d_out + i];
            uint16_t hb = 0;
            if (isfinite(p))
                hb = __half_as_ushort(__float2half_rn(p));
            else
                st |= BITSMOE_ST_NONFINITE;
            w16[i] = hb;
        }
    } else {
        QGroup q = qgroup(blob, d, item.g);
        uint32_t* planes = const_cast<uint32_t*>(q.planes);
        switch (group_width(item.g)) {
            case 8: pack_word<8>(comps_e, q.idx, q.scale, q.n, item.w, q.W, d_out, d_pad, planes, st); break;
            case 6: pack_word<6>(comps_e, q.idx, q.scale, q.n, item.w, q.W, d_out, d_pad, planes, st); break;
            case 4: pack_word<4>(comps_e, q.idx, q.scale, q.n, item.w, q.W, d_out, d_pad, planes, st); break;
            case 3: pack_word<3>(comps_e, q.idx, q.scale, q.n, item.w, q.W, d_out, d_pad, planes, st); break;
            case 2: pack_word<2>(comps_e, q.idx, q.scale, q.n, item.w, q.W, d_out, d_pad, planes, st); break;
            case 1: pack_word<1>(comps_e, q.idx, q.scale, q.n, item.w, q.W, d_out, d_pad, planes, st); break;
        }
    }
    }
    if (st && status) atomicOr(status, st);
}

// ---------------------------------------------------------------------------
// unpack (test support)
// ---------------------------------------------------------------------------
__global__ void k_unpack(const uint8_t* __restrict__ blob, uint16_t* __restrict__ qout, int r, int d_out,
                         uint32_t d_pad) {
    const int e = blockIdx.x;
    const DirEntry d = read_dir(blob, e);
    uint16_t* q_e = qout + (uint64_t)e * r * d_out;
    Item item;
    for (uint32_t it = blockIdx.y; item_of(d, it, item); it += gridDim.y) {
    if (item.g == 0) {
        HGroup h = hgroup(blob, d);
        uint32_t k = h.idx[item.w];
        for (uint32_t i = blockIdx.z * blockDim.x + threadIdx.x; i < (uint32_t)d_out; i += gridDim.z * blockDim.x)
            q_e[(uint64_t)k * d_out + i] = h.w16[(uint64_t)item.w * d_pad + i];
        continue;
    }
    QGroup q = qgroup(blob, d, item.g);
    const int b = group_width(item.g);
    const uint32_t valid = min(32u, q.n - 32 * item.w);
    for (uint32_t i = blockIdx.z * blockDim.x + threadIdx.x; i < (uint32_t)d_out; i += gridDim.z * blockDim.x) {
        uint32_t word[8];
        for (int j = 0; j < b; j++) word[j] = q.planes[plane_word(j, item.w, q.W, d_pad, i)];
        for (uint32_t m = 0; m < valid; m++) {
            uint32_t v = 0;
            for (int j = 0; j < b; j++) v |= ((word[j] >> m) & 1u) << j;
            q_e[(uint64_t)q.idx[32 * item.w + m] * d_out + i] = (uint16_t)v;
        }
    }
    }
}

static dim3 item_grid(const bitsmoe_plan* p) {
    uint32_t zb = (uint32_t)((p->dims.d_out + 255) / 256);
    if (zb > 64) zb = 64;
    uint32_t yb = p->max_items ? p->max_items : 1;
    if (yb > 65535) yb = 65535;
    return dim3((unsigned)p->dims.n_experts, yb, zb);
}

}  // namespace bitsmoe

using namespace bitsmoe;

BITSMOE_API int bitsmoe_compute_scales(const bitsmoe_plan* plan, const float* comps, const uint8_t* widths,
                                       uint16_t* scales, int32_t* status, void* stream) {
    if (!plan || !comps || !widths || !scales) return BITSMOE_EINVAL;
    uint64_t n = (uint64_t)plan->dims.n_experts * plan->dims.rank;
    uint64_t blocks = (n * 32 + 255) / 256;
    k_compute_scales<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(comps, widths, scales, status, n,
                                                                        plan->dims.d_out);
    return check_launch();
}

BITSMOE_API int bitsmoe_pack(const bitsmoe_plan* plan, const float* comps, const uint8_t* widths,
                             const uint16_t* scales, const float* amps, void* blob, int32_t* status, void* stream) {
    if (!plan || !comps || !widths || !scales || !amps || !blob) return BITSMOE_EINVAL;
    if ((uintptr_t)blob % 16) return BITSMOE_EINVAL;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(blob, 0, plan->blob_bytes, s);
    if (e != cudaSuccess) return set_cuda_error(e);
    e = cudaMemcpyAsync(blob, plan->header, plan->header_bytes, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return set_cuda_error(e);
    const int r = plan->dims.rank;
    if ((size_t)r > 48 * 1024) {
        e = cudaFuncSetAttribute(k_pack_index, cudaFuncAttributeMaxDynamicSharedMemorySize, r);
        if (e != cudaSuccess) return set_cuda_error(e);
    }
    k_pack_index<<<plan->dims.n_experts, kIndexThreads, r, s>>>(widths, scales, amps, (uint8_t*)blob, r, status);
    int rc = check_launch();
    if (rc) return rc;
    if (plan->max_items == 0) return BITSMOE_OK;
    k_pack_planes<<<item_grid(plan), 256, 0, s>>>(comps, (uint8_t*)blob, r, plan->dims.d_out, plan->d_pad, status);
    return check_launch();
}

BITSMOE_API int bitsmoe_unpack_q(const bitsmoe_plan* plan, const void* blob, uint16_t* q, void* stream) {
    if (!plan || !blob || !q) return BITSMOE_EINVAL;
    cudaStream_t s = (cudaStream_t)stream;
    uint64_t n = (uint64_t)plan->dims.n_experts * plan->dims.rank * plan->dims.d_out;
    cudaError_t e = cudaMemsetAsync(q, 0, n * sizeof(uint16_t), s);
    if (e != cudaSuccess) return set_cuda_error(e);
    if (plan->max_items == 0) return BITSMOE_OK;
    k_unpack<<<item_grid(plan), 256, 0, s>>>((const uint8_t*)blob, q, plan->dims.rank, plan->dims.d_out,
                                             plan->d_pad);
    return check_launch();
}
