// expert.cu -- routed expert forward over width-grouped bit planes, the routed
// combine, and the general (any T) layer forward built from them.
//
// Per routed (token t, slot j) with expert e (BitsMoE study-note page,
// Methodology: W_e x = P_e A_e (Phi^T x); second split: unit directions with
// amplitudes; Execution: bit planes grouped by width):
//   Y_e[t][j][i] = sum_b ( sum_bit 2^bit sum_{k in G_b} c_k bit_{k,bit,i}
//                          - (2^b - 1)/2 sum_{k in G_b} c_k )
//                + sum_{k in G_16} a_k z_k w16_{k,i},       c_k = a_k s_k z_{t,k}
// Tokens routed to the same expert are grouped first, so each expert's planes
// are streamed once per call however many of the batch's tokens use it.
#include <algorithm>

#include "common.cuh"

namespace bitsmoe {

int launch_shared_proj(const uint16_t* phi_t, const uint16_t* X, float* Z, int T, int d_in, int r, cudaStream_t s);

// ---------------------------------------------------------------------------
// workspace layout
// ---------------------------------------------------------------------------

struct WsCursor {
    uint8_t* p;
    uint64_t used;
    void* take(uint64_t bytes) {
        uint64_t off = roundup(used, 256);
        used = off + bytes;
        return p ? p + off : nullptr;
    }
};

uint32_t cvals_ldc(const bitsmoe_plan* p);

static RouteWS take_route(WsCursor& c, int E, int T, int K, uint32_t ldc) {
    RouteWS r;
    r.count = (int32_t*)c.take(4ull * E);
    r.start = (int32_t*)c.take(4ull * (E + 1));
    r.active = (int32_t*)c.take(4ull * E);
    r.nactive = (int32_t*)c.take(4);
    r.pairs = (int32_t*)c.take(4ull * (uint64_t)T * K + 4);
    r.ldc = ldc;
    r.cvals = (float*)c.take(4ull * (uint64_t)T * K * ldc);
    r.zp = (float*)c.take(4ull * (uint64_t)T * K + 4);
    return r;
}

// ---------------------------------------------------------------------------
// routing groups: one CTA
// ---------------------------------------------------------------------------
constexpr int kRouteThreads = 1024;

__global__ void __launch_bounds__(kRouteThreads) k_route(const int32_t* __restrict__ ids, int npairs, int E,
                                                         RouteWS ws, int32_t* status) {
    __shared__ int32_t s_part[kRouteThreads], s_apart[kRouteThreads];
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += blockDim.x) ws.count[e] = 0;
    __syncthreads();
    bool bad = false;
    for (int p = tid; p < npairs; p += blockDim.x) {
        int e = ids[p];
        if (e < 0 || e >= E)
            bad = true;
        else
            atomicAdd(&ws.count[e], 1);
    }
    if (bad && status) atomicOr(status, BITSMOE_ST_BADEXPERT);
    __syncthreads();
    // exclusive scans of count (-> start) and of (count > 0) (-> active list)
    const int chunk = (E + blockDim.x - 1) / blockDim.x;
    const int e0 = min(E, tid * chunk), e1 = min(E, e0 + chunk);
    int sum = 0, asum = 0;
    for (int e = e0; e < e1; e++) {
        int c = ws.count[e];
        sum += c;
        asum += c > 0;
    }
    s_part[tid] = sum;
    s_apart[tid] = asum;
    __syncthreads();
    for (int o = 1; o < (int)blockDim.x; o <<= 1) {  // inclusive Hillis-Steele
        int v = tid >= o ? s_part[tid - o] : 0;
        int a = tid >= o ? s_apart[tid - o] : 0;
        __syncthreads();
        s_part[tid] += v;
        s_apart[tid] += a;
        __syncthreads();
    }
    int run = s_part[tid] - sum, arun = s_apart[tid] - asum;
    for (int e = e0; e < e1; e++) {
        int c = ws.count[e];
        ws.start[e] = run;
        if (c > 0) ws.active[arun++] = e;
        ws.count[e] = run;  // becomes the scatter cursor
        run += c;
    }
    if (tid == blockDim.x - 1) {
        ws.start[E] = s_part[tid];
        *ws.nactive = s_apart[tid];
    }
    __syncthreads();
    for (int p = tid; p < npairs; p += blockDim.x) {
        int e = ids[p];
        if (e >= 0 && e < E) ws.pairs[atomicAdd(&ws.count[e], 1)] = p;
    }
}

// Y_sum[t][i] = sum_j g[t][j] Y_e[t][j][i]; rows of out-of-range ids are zeroed.
__global__ void k_combine(const int32_t* __restrict__ ids, const float* __restrict__ gw, float* Ye,
                          float* __restrict__ Ysum, int T, int K, int E, int d_out) {
    uint64_t n = (uint64_t)T * d_out;
    for (uint64_t x = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n; x += (uint64_t)gridDim.x * blockDim.x) {
        uint64_t t = x / d_out, i = x % d_out;
        float acc = 0.0f;
        for (int j = 0; j < K; j++) {
            int e = ids[t * K + j];
            float* y = Ye + (t * K + j) * (uint64_t)d_out + i;
            if (e < 0 || e >= E) {
                *y = 0.0f;
                continue;
            }
            acc = fmaf(gw[t * K + j], *y, acc);
        }
        Ysum[x] = acc;
    }
}

int launch_expert_mt(const bitsmoe_plan* p, const void* blob, const float* Z, const int32_t* ids, int T,
                     const RouteWS& rw, float* Ye, int32_t* status, cudaStream_t s);

static int launch_expert(const bitsmoe_plan* p, const void* blob, const float* Z, const int32_t* ids,
                         const float* gw, int T, float* Ye, float* Ysum, const RouteWS& rw, int32_t* status,
                         cudaStream_t s) {
    const int E = p->dims.n_experts, K = p->dims.top_k, d_out = p->dims.d_out;
    int rc = launch_expert_mt(p, blob, Z, ids, T, rw, Ye, status, s);
    if (rc) return rc;
    uint64_t n = (uint64_t)T * d_out;
    unsigned blocks = (unsigned)std::min<uint64_t>((n + 255) / 256, 4096);
    k_combine<<<blocks, 256, 0, s>>>(ids, gw, Ye, Ysum, T, K, E, d_out);
    return check_launch();
}

static int launch_route(const bitsmoe_plan* p, const int32_t* ids, int T, const RouteWS& rw, int32_t* status,
                        cudaStream_t s) {
    k_route<<<1, kRouteThreads, 0, s>>>(ids, T * p->dims.top_k, p->dims.n_experts, rw, status);
    return check_launch();
}

// Routing groups of npairs (token, slot) pairs and the slot-order routed sum, for
// the other steps of the library that group tokens by expert (the down projection).
int launch_route_ids(const int32_t* ids, int npairs, int E, const RouteWS& rw, int32_t* status, cudaStream_t s) {
    k_route<<<1, kRouteThreads, 0, s>>>(ids, npairs, E, rw, status);
    return check_launch();
}
int launch_combine(const int32_t* ids, const float* gw, float* Ye, float* Ysum, int T, int K, int E, int d_out,
                   cudaStream_t s) {
    const uint64_t n = (uint64_t)T * d_out;
    const unsigned blocks = (unsigned)std::min<uint64_t>((n + 255) / 256, 4096);
    k_combine<<<blocks, 256, 0, s>>>(ids, gw, Ye, Ysum, T, K, E, d_out);
    return check_launch();
}

static uint64_t expert_ws(const bitsmoe_plan* p, int T, bool need_ye, uint8_t* base, RouteWS* rw, float** ye) {
    WsCursor c{base, 0};
    RouteWS r = take_route(c, p->dims.n_experts, T, p->dims.top_k, cvals_ldc(p));
    float* y = need_ye ? (float*)c.take(4ull * T * p->dims.top_k * p->dims.d_out) : nullptr;
    if (rw) *rw = r;
    if (ye) *ye = y;
    return c.used;
}

}  // namespace bitsmoe

using namespace bitsmoe;

BITSMOE_API uint64_t bitsmoe_expert_workspace_bytes(const bitsmoe_plan* plan, int32_t T) {
    if (!plan || T < 0) return 0;
    return expert_ws(plan, T, true, nullptr, nullptr, nullptr);
}

BITSMOE_API int bitsmoe_expert_forward(const bitsmoe_plan* plan, const void* blob, const float* Z,
                                       const int32_t* topk_ids, const float* gate_w, int32_t T, float* Y_experts,
                                       float* Y_sum, void* workspace, uint64_t workspace_bytes, int32_t* status,
                                       void* stream) {
    if (!plan || T < 0) return BITSMOE_EINVAL;
    if (T == 0) return BITSMOE_OK;
    if (!blob || !Z || !topk_ids || !gate_w || !Y_sum || !workspace) return BITSMOE_EINVAL;
    if ((uintptr_t)blob % 16 || (uintptr_t)workspace % 256) return BITSMOE_EINVAL;
    if (workspace_bytes < bitsmoe_expert_workspace_bytes(plan, T)) return BITSMOE_ESIZE;
    RouteWS rw;
    float* ye_ws;
    expert_ws(plan, T, Y_experts == nullptr, (uint8_t*)workspace, &rw, &ye_ws);
    float* Ye = Y_experts ? Y_experts : ye_ws;
    cudaStream_t s = (cudaStream_t)stream;
    int rc = launch_route(plan, topk_ids, T, rw, status, s);
    if (rc) return rc;
    return launch_expert(plan, blob, Z, topk_ids, gate_w, T, Ye, Y_sum, rw, status, s);
}

// ---------------------------------------------------------------------------
// layer forward (both projections)
// ---------------------------------------------------------------------------
namespace bitsmoe {
struct LayerWS {
    RouteWS route;
    float* Z[2];
    float* Ye[2];
};
static uint64_t layer_ws(const bitsmoe_plan* g, const bitsmoe_plan* u, int T, const bitsmoe_proj_io* io[2],
                         uint8_t* base, LayerWS* out) {
    WsCursor c{base, 0};
    LayerWS L;
    L.route = take_route(c, g->dims.n_experts, T, g->dims.top_k, std::max(cvals_ldc(g), cvals_ldc(u)));
    const bitsmoe_plan* p[2] = {g, u};
    for (int j = 0; j < 2; j++) {
        L.Z[j] = (!io || !io[j]->Z) ? (float*)c.take(4ull * T * p[j]->dims.rank) : nullptr;
        L.Ye[j] = (!io || !io[j]->Y_experts) ? (float*)c.take(4ull * T * p[j]->dims.top_k * p[j]->dims.d_out) : nullptr;
    }
    if (out) *out = L;
    return c.used;
}

int layer_forward_fused_t1(const bitsmoe_proj_io* io[2], const uint16_t* X, const int32_t* ids, const float* gw,
                           void* workspace, uint64_t workspace_bytes, const uint16_t* const* next_phi, int32_t* status,
                           cudaStream_t s, bool* used);
uint64_t layer_fused_t1_reserved(const bitsmoe_plan* g, const bitsmoe_plan* u);
}  // namespace bitsmoe

// Layer workspace = [fused single-token path's state (persistent) | per-call region of the other paths].
BITSMOE_API uint64_t bitsmoe_layer_workspace_bytes(const bitsmoe_plan* gate, const bitsmoe_plan* up, int32_t T) {
    if (!gate || !up || T < 0) return 0;
    const uint64_t head = layer_fused_t1_reserved(gate, up);
    return head + layer_ws(gate, up, T, nullptr, nullptr, nullptr);
}

BITSMOE_API int bitsmoe_layer_launches(const bitsmoe_plan* gate, const bitsmoe_plan* up, int32_t T) {
    if (!gate || !up || T < 0) return BITSMOE_EINVAL;
    if (T == 0) return 0;
    if (T == 1 && layer_fused_t1_reserved(gate, up) > 0) return 1;
    return 7;  // route, then per projection: shared projection, experts, combine
}

static int layer_forward_impl(const bitsmoe_proj_io* gate, const bitsmoe_proj_io* up, const uint16_t* X,
                              const int32_t* topk_ids, const float* gate_w, int32_t T, void* workspace,
                              uint64_t workspace_bytes, const uint16_t* const* next_phi, int32_t* status, void* stream) {
    if (!gate || !up || T < 0 || !gate->plan || !up->plan) return BITSMOE_EINVAL;
    const bitsmoe_proj_io* io[2] = {gate, up};
    const bitsmoe_plan *pg = gate->plan, *pu = up->plan;
    if (pg->dims.d_in != pu->dims.d_in || pg->dims.top_k != pu->dims.top_k ||
        pg->dims.n_experts != pu->dims.n_experts)
        return BITSMOE_EINVAL;
    if (pg->dims.d_in % 8) return BITSMOE_EINVAL;
    if (T == 0) return BITSMOE_OK;
    for (int j = 0; j < 2; j++) {
        if (!io[j]->blob || !io[j]->phi_t || !io[j]->Y_sum) return BITSMOE_EINVAL;
        if ((uintptr_t)io[j]->blob % 16 || (uintptr_t)io[j]->phi_t % 16) return BITSMOE_EINVAL;
    }
    if (!X || !topk_ids || !gate_w || !workspace) return BITSMOE_EINVAL;
    if ((uintptr_t)X % 16 || (uintptr_t)workspace % 256) return BITSMOE_EINVAL;
    if (workspace_bytes < bitsmoe_layer_workspace_bytes(pg, pu, T)) return BITSMOE_ESIZE;
    cudaStream_t s = (cudaStream_t)stream;
    if (T == 1) {
        bool used = false;
        int rc = layer_forward_fused_t1(io, X, topk_ids, gate_w, workspace, workspace_bytes, next_phi, status, s, &used);
        if (rc || used) return rc;
    }
    LayerWS L;
    layer_ws(pg, pu, T, io, (uint8_t*)workspace + layer_fused_t1_reserved(pg, pu), &L);
    int rc = launch_route(pg, topk_ids, T, L.route, status, s);
    if (rc) return rc;
    for (int j = 0; j < 2; j++) {
        const bitsmoe_plan* p = io[j]->plan;
        float* Z = io[j]->Z ? io[j]->Z : L.Z[j];
        float* Ye = io[j]->Y_experts ? io[j]->Y_experts : L.Ye[j];
        rc = launch_shared_proj(io[j]->phi_t, X, Z, T, p->dims.d_in, p->dims.rank, s);
        if (rc) return rc;
        rc = launch_expert(p, io[j]->blob, Z, topk_ids, gate_w, T, Ye, io[j]->Y_sum, L.route, status, s);
        if (rc) return rc;
    }
    return BITSMOE_OK;
}

BITSMOE_API int bitsmoe_layer_forward(const bitsmoe_proj_io* gate, const bitsmoe_proj_io* up, const uint16_t* X,
                                      const int32_t* topk_ids, const float* gate_w, int32_t T, void* workspace,
                                      uint64_t workspace_bytes, int32_t* status, void* stream) {
    return layer_forward_impl(gate, up, X, topk_ids, gate_w, T, workspace, workspace_bytes, nullptr, status, stream);
}

BITSMOE_API int bitsmoe_layer_forward_chained(const bitsmoe_proj_io* gate, const bitsmoe_proj_io* up,
                                              const uint16_t* X, const int32_t* topk_ids, const float* gate_w,
                                              int32_t T, void* workspace, uint64_t workspace_bytes,
                                              const uint16_t* next_phi_t_gate, const uint16_t* next_phi_t_up,
                                              int32_t* status, void* stream) {
    if ((next_phi_t_gate == nullptr) != (next_phi_t_up == nullptr)) return BITSMOE_EINVAL;
    if ((uintptr_t)next_phi_t_gate % 16 || (uintptr_t)next_phi_t_up % 16) return BITSMOE_EINVAL;
    const uint16_t* next[2] = {next_phi_t_gate, next_phi_t_up};
    return layer_forward_impl(gate, up, X, topk_ids, gate_w, T, workspace, workspace_bytes,
                              next_phi_t_gate ? next : nullptr, status, stream);
}

// ---------------------------------------------------------------------------
// the whole expert FFN: the layer (gate and up), then the down step
// ---------------------------------------------------------------------------
BITSMOE_API uint64_t bitsmoe_ffn_workspace_bytes(const bitsmoe_plan* gate, const bitsmoe_plan* up, int32_t T) {
    if (!gate || !up || T < 0) return 0;
    const bitsmoe_ffn_dims d{gate->dims.d_in, gate->dims.d_out, gate->dims.n_experts, gate->dims.top_k};
    return roundup(bitsmoe_layer_workspace_bytes(gate, up, T), 256) + bitsmoe_ffn_down_workspace_bytes(&d, T);
}

BITSMOE_API int bitsmoe_ffn_launches(const bitsmoe_plan* gate, const bitsmoe_plan* up, int32_t T) {
    if (!gate || !up || T < 0) return BITSMOE_EINVAL;
    const bitsmoe_ffn_dims d{gate->dims.d_in, gate->dims.d_out, gate->dims.n_experts, gate->dims.top_k};
    const int nl = bitsmoe_layer_launches(gate, up, T), nd = bitsmoe_ffn_down_launches(&d, T);
    if (nl < 0) return nl;
    if (nd < 0) return nd;
    return nl + nd;
}

BITSMOE_API int bitsmoe_ffn_forward(const bitsmoe_proj_io* gate, const bitsmoe_proj_io* up, const uint16_t* w_down,
                                    const uint16_t* X, const int32_t* topk_ids, const float* gate_w, int32_t T,
                                    float* out, void* workspace, uint64_t workspace_bytes, int32_t* status,
                                    void* stream) {
    if (!gate || !up || !gate->plan || !up->plan || T < 0) return BITSMOE_EINVAL;
    const bitsmoe_plan *pg = gate->plan, *pu = up->plan;
    if (pg->dims.d_out != pu->dims.d_out) return BITSMOE_EINVAL;
    const bitsmoe_ffn_dims d{pg->dims.d_in, pg->dims.d_out, pg->dims.n_experts, pg->dims.top_k};
    if (T == 0) return BITSMOE_OK;
    if (!gate->Y_experts || !up->Y_experts || !w_down || !out || !workspace) return BITSMOE_EINVAL;
    if ((uintptr_t)w_down % 16 || (uintptr_t)gate->Y_experts % 16 || (uintptr_t)up->Y_experts % 16) return BITSMOE_EINVAL;
    if (d.d_ff % 8) return BITSMOE_EINVAL;
    if (workspace_bytes < bitsmoe_ffn_workspace_bytes(pg, pu, T)) return BITSMOE_ESIZE;
    const uint64_t lw = bitsmoe_layer_workspace_bytes(pg, pu, T), off = roundup(lw, 256);
    int rc = layer_forward_impl(gate, up, X, topk_ids, gate_w, T, workspace, lw, nullptr, status, stream);
    if (rc) return rc;
    return bitsmoe_ffn_down(&d, w_down, gate->Y_experts, up->Y_experts, topk_ids, gate_w, T, out,
                            (uint8_t*)workspace + off, workspace_bytes - off, status, stream);
}
