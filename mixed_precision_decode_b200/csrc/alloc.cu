// alloc.cu -- the allocation of widths (offline, host): the FQCM cost of every
// component at every width, and the choice of widths under a bit budget
// (BitsMoE study-note page, Methodology, third split: activation-dependent
// importance beta_{e,k} = phi_k^T X_e G_e X_e^T phi_k = sum_j g_{e,j} (phi_k^T x_j)^2,
// importance I = a_{e,k}^2 beta_{e,k}, cost L_{e,k}(b) = I eps_{e,k,b}; the gain of
// more bits per stored bit, a component of m elements costing m (b' - b) more
// bits; Usage: an integer program over the width set {0,1,2,3,4,6,8,16} under a
// bit budget, every candidate width of every component considered jointly).
//
// eps_{e,k,b} is not defined on the pages: it is taken as the squared error of
// storing the unit direction p_{e,k} at width b with this library's quantiser
// (one fp16 scale s = fp16(2 max|p| / (2^b - 1)), q = clamp(floor(p/s + 2^(b-1))),
// stored w = s (q - (2^b - 1)/2)); 16 bits store fp16(p), 0 bits nothing.
//
// The integer program is solved through its linear relaxation, which for this
// multiple-choice knapsack has a direct solution: per component, the lower convex
// hull of its (bits, loss) points from width 0; then all hull segments of all
// components in order of loss saved per bit, each taken while it fits the budget
// and the first that does not fit ending the allocation.  Where the relaxation's
// solution is integral (budgets at its vertices) it is the integer optimum.
//
// Every step runs on the host in fp64 in a fixed order (threads split independent
// components or experts), so the results do not depend on the thread count.
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <thread>
#include <vector>

#include "common.cuh"

namespace bitsmoe {

static const int kWidthSet[8] = {0, 1, 2, 3, 4, 6, 8, 16};  // the order of eps arrays

// Runs f(i0, i1) over [0, n) split into contiguous ranges on host threads.
template <typename F>
static void parallel_ranges(int64_t n, F f) {
    const int64_t nt = std::max<int64_t>(1, std::min<int64_t>({(int64_t)std::thread::hardware_concurrency(), 32, n}));
    std::vector<std::thread> pool;
    for (int64_t t = 1; t < nt; t++) pool.emplace_back(f, n * t / nt, n * (t + 1) / nt);
    f(0, n / nt);
    for (auto& th : pool) th.join();
}

// eps at every width of kWidthSet for one direction p (d_out elements, largest
// magnitude m, all finite), in one pass over p: per element, every width's stored
// value and squared error, each width's sum taken in element order in fp64.
static void eps_all(const float* p, int d_out, float m, double* out) {
    constexpr int kQ = 6;  // the widths with a scale: 1, 2, 3, 4, 6, 8
    float s[kQ], half[kQ], qmax[kQ];
    double mid[kQ], acc[kQ];
    bool stores[kQ];
    for (int j = 0; j < kQ; j++) {
        const int b = kWidthSet[1 + j];
        s[j] = __half2float(__float2half_rn((2.0f * m) / (float)((1 << b) - 1)));
        stores[j] = std::isfinite(s[j]) && s[j] > 0.0f;  // else every q is 0
        half[j] = (float)(1 << (b - 1));
        qmax[j] = (float)((1 << b) - 1);
        mid[j] = (double)((1 << b) - 1) / 2.0;
        acc[j] = 0.0;
    }
    double acc0 = 0.0, acc16 = 0.0;
    for (int i = 0; i < d_out; i++) {
        const float x = p[i];
        const double xd = (double)x;
        acc0 += xd * xd;  // 0 bits: nothing stored
        const double d16 = xd - (double)__half2float(__float2half_rn(x));  // 16 bits: fp16(p)
        acc16 += d16 * d16;
        for (int j = 0; j < kQ; j++) {
            float q = 0.0f;
            if (stores[j]) {
                // t = x / s and u = t + 2^(b-1) as separate fp32 operations; for u >= 0
                // the integer part is floor(u), and past the top level the clamp applies
                const float u = x / s[j] + half[j];
                q = u < 0.0f ? 0.0f : (float)(int)std::min(u, qmax[j]);
            }
            const double d = xd - (double)s[j] * ((double)q - mid[j]);
            acc[j] += d * d;
        }
    }
    out[0] = acc0;
    for (int j = 0; j < kQ; j++) out[1 + j] = acc[j];
    out[7] = acc16;
}

}  // namespace bitsmoe

using namespace bitsmoe;

BITSMOE_API int bitsmoe_fqcm_eps(const float* comps, int32_t E, int32_t r, int32_t d_out, double* eps) {
    if (!comps || !eps || E < 1 || r < 1 || d_out < 1) return BITSMOE_EINVAL;
    parallel_ranges((int64_t)E * r, [&](int64_t c0, int64_t c1) {
        for (int64_t c = c0; c < c1; c++) {
            const float* p = comps + (size_t)c * d_out;
            double* out = eps + (size_t)c * 8;
            float m = 0.0f;
            bool bad = false;
            for (int i = 0; i < d_out; i++) {
                if (!std::isfinite(p[i])) bad = true;
                m = std::max(m, std::fabs(p[i]));
            }
            if (bad)
                for (int wi = 0; wi < 8; wi++) out[wi] = NAN;
            else
                eps_all(p, d_out, m, out);
        }
    });
    return BITSMOE_OK;
}

BITSMOE_API int bitsmoe_fqcm_beta(const float* Z, const int32_t* topk_ids, const float* gate_w, int32_t T,
                                  int32_t top_k, int32_t E, int32_t r, double* beta) {
    if (T < 0 || top_k < 1 || E < 1 || r < 1 || !beta) return BITSMOE_EINVAL;
    if (T > 0 && (!Z || !topk_ids || !gate_w)) return BITSMOE_EINVAL;
    // experts are independent: each thread owns a range of experts and walks all pairs
    parallel_ranges(E, [&](int64_t e0, int64_t e1) {
        for (int64_t e = e0; e < e1; e++) std::fill(beta + (size_t)e * r, beta + (size_t)(e + 1) * r, 0.0);
        for (int t = 0; t < T; t++)
            for (int j = 0; j < top_k; j++) {
                const int e = topk_ids[(size_t)t * top_k + j];
                if (e < e0 || e >= e1) continue;
                const double g = (double)gate_w[(size_t)t * top_k + j];
                const float* z = Z + (size_t)t * r;
                double* b = beta + (size_t)e * r;
                for (int k = 0; k < r; k++) {
                    const double zk = (double)z[k];
                    b[k] += g * (zk * zk);
                }
            }
    });
    return BITSMOE_OK;
}

namespace {
struct Seg {
    double eff;    // loss saved per bit
    int64_t c;     // component e * r + k
    int s;         // position on the component's hull
    int64_t cost;  // bits
    int wi;        // the width index this segment reaches
};
}  // namespace

// The lower convex hull of one component's (bits, loss) points from width 0, as
// segments (out: up to 7), or none when its cost is not finite.
static int hull_segments(int64_t c, double a, double beta, const double* eps8, int d_out, Seg* out) {
    struct Pt {
        int64_t bits;
        double loss;
        int wi;
    };
    const double imp = a * a * beta;
    bool finite = std::isfinite(imp);
    for (int wi = 0; wi < 8; wi++) finite = finite && std::isfinite(eps8[wi]);
    if (!finite) return 0;  // a component without a finite cost keeps width 0
    Pt hull[8];
    int h = 0;
    hull[h++] = {0, imp * eps8[0], 0};
    for (int wi = 1; wi < 8; wi++) {
        const Pt pt{(int64_t)d_out * kWidthSet[wi], imp * eps8[wi], wi};
        if (pt.loss >= hull[h - 1].loss) continue;  // more bits and no less loss
        while (h >= 2) {
            const Pt& A = hull[h - 2];
            const Pt& Bq = hull[h - 1];
            if ((Bq.loss - A.loss) * (double)(pt.bits - A.bits) >= (pt.loss - A.loss) * (double)(Bq.bits - A.bits))
                h--;
            else
                break;
        }
        hull[h++] = pt;
    }
    for (int s = 0; s + 1 < h; s++) {
        const double gain = hull[s].loss - hull[s + 1].loss;
        const int64_t cost = hull[s + 1].bits - hull[s].bits;
        out[s] = {gain / (double)cost, c, s, cost, hull[s + 1].wi};
    }
    return h - 1;
}

static bool seg_before(const Seg& x, const Seg& y) {
    if (x.eff != y.eff) return x.eff > y.eff;
    if (x.c != y.c) return x.c < y.c;
    return x.s < y.s;
}

BITSMOE_API int bitsmoe_allocate_widths(const float* amps, const double* beta, const double* eps, int32_t E,
                                        int32_t r, int32_t d_out, uint64_t budget_bits, uint8_t* widths,
                                        double* loss_out) {
    if (!amps || !beta || !eps || !widths || E < 1 || r < 1 || d_out < 1) return BITSMOE_EINVAL;
    const int64_t n = (int64_t)E * r;
    // every component's hull segments into one array: count, offsets, then fill
    std::vector<uint8_t> nseg((size_t)n);
    parallel_ranges(n, [&](int64_t c0, int64_t c1) {
        Seg tmp[7];
        for (int64_t c = c0; c < c1; c++)
            nseg[(size_t)c] = (uint8_t)hull_segments(c, (double)amps[c], beta[c], eps + (size_t)c * 8, d_out, tmp);
    });
    std::vector<int64_t> off((size_t)n + 1, 0);
    for (int64_t c = 0; c < n; c++) off[(size_t)c + 1] = off[(size_t)c] + nseg[(size_t)c];
    std::vector<Seg> segs((size_t)off[(size_t)n]);
    parallel_ranges(n, [&](int64_t c0, int64_t c1) {
        for (int64_t c = c0; c < c1; c++)
            hull_segments(c, (double)amps[c], beta[c], eps + (size_t)c * 8, d_out, segs.data() + off[(size_t)c]);
    });
    // sorted by loss saved per bit (a strict total order: the result does not depend on
    // how the sort is split): runs sorted on host threads, then merged pairwise
    const int64_t m = (int64_t)segs.size();
    const int64_t nt = std::max<int64_t>(1, std::min<int64_t>({(int64_t)std::thread::hardware_concurrency(), 16,
                                                               m / 4096 + 1}));
    std::vector<int64_t> bound((size_t)nt + 1);
    for (int64_t t = 0; t <= nt; t++) bound[(size_t)t] = m * t / nt;
    parallel_ranges(nt, [&](int64_t t0, int64_t t1) {
        for (int64_t t = t0; t < t1; t++)
            std::sort(segs.begin() + bound[(size_t)t], segs.begin() + bound[(size_t)t + 1], seg_before);
    });
    for (int64_t width = 1; width < nt; width *= 2) {
        std::vector<std::thread> pool;
        for (int64_t t = 0; t + width < nt; t += 2 * width) {
            const int64_t a = bound[(size_t)t], mid = bound[(size_t)(t + width)],
                          b = bound[(size_t)std::min(nt, t + 2 * width)];
            pool.emplace_back([&segs, a, mid, b] {
                std::inplace_merge(segs.begin() + a, segs.begin() + mid, segs.begin() + b, seg_before);
            });
        }
        for (auto& th : pool) th.join();
    }
    std::vector<uint8_t> choice((size_t)n, 0);
    uint64_t used = 0;
    for (const Seg& sg : segs) {
        if (used + (uint64_t)sg.cost > budget_bits) break;
        used += (uint64_t)sg.cost;
        choice[(size_t)sg.c] = (uint8_t)sg.wi;
    }
    double loss = 0.0;
    for (int64_t c = 0; c < n; c++) {
        widths[c] = (uint8_t)kWidthSet[choice[(size_t)c]];
        const double a = (double)amps[c];
        loss += a * a * beta[c] * eps[(size_t)c * 8 + choice[(size_t)c]];
    }
    if (loss_out) *loss_out = loss;
    return BITSMOE_OK;
}
