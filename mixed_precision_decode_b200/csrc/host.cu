// host.cu -- plans, argument checks, error text and status read-back.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"

namespace bitsmoe {

static thread_local char g_cuda_msg[256] = "no CUDA error recorded";

int set_cuda_error(cudaError_t e) {
    snprintf(g_cuda_msg, sizeof(g_cuda_msg), "CUDA error %d: %s", (int)e, cudaGetErrorString(e));
    return BITSMOE_ECUDA;
}

int check_launch() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? BITSMOE_OK : set_cuda_error(e);
}

static void put16(uint8_t* p, uint16_t v) { memcpy(p, &v, 2); }
static void put32(uint8_t* p, uint32_t v) { memcpy(p, &v, 4); }
static void put64(uint8_t* p, uint64_t v) { memcpy(p, &v, 8); }
static uint16_t get16(const uint8_t* p) { uint16_t v; memcpy(&v, p, 2); return v; }
static uint32_t get32(const uint8_t* p) { uint32_t v; memcpy(&v, p, 4); return v; }

static bool dims_ok(const bitsmoe_dims* d) {
    return d && d->d_in >= 1 && d->d_out >= 1 && d->d_out <= (1 << 30) && d->n_experts >= 1 &&
           d->n_experts <= (1 << 20) && d->rank >= 1 && d->rank <= 65535 && d->top_k >= 1 && d->top_k <= 1024;
}

// Fills sizes, the header image and the derived launch bounds from counts.
static int finish_plan(bitsmoe_plan* p) {
    const int E = p->dims.n_experts;
    p->d_pad = (uint32_t)roundup((uint64_t)p->dims.d_out, 32);
    p->header_bytes = kHeaderBytes + kDirEntryBytes * (uint64_t)E;
    p->header = (uint8_t*)calloc(p->header_bytes, 1);
    if (!p->header) return BITSMOE_ENOMEM;
    uint64_t base = p->header_bytes;
    p->max_items = 0;
    p->max_members_padded = 0;
    p->max_t1_items = 0;
    for (int e = 0; e < E; e++) {
        const uint32_t* c = p->counts + 8 * (size_t)e;
        uint8_t* dir = p->header + kHeaderBytes + kDirEntryBytes * (uint64_t)e;
        uint64_t off = 0;
        uint32_t items = 0, members = 0, t1_items = 0;
        for (int g = 0; g < kNumGroups; g++) {
            int b = group_width(g);
            put32(dir + 16 + 4 * g, (uint32_t)off);
            put16(dir + 44 + 2 * g, (uint16_t)c[g]);
            off += group_bytes(b, c[g], p->d_pad);
            uint32_t np = (uint32_t)group_members_padded(b, c[g]);
            members += np;
            items += b == 16 ? c[g] : np / 32;
            t1_items += b == 16 ? np / 8 : b * (np / 32);  // fp16 members padded to octets
        }
        put16(dir + 44 + 14, (uint16_t)c[7]);
        put64(dir, base);
        put64(dir + 8, off);
        base += off;
        if (items > p->max_items) p->max_items = items;
        if (members > p->max_members_padded) p->max_members_padded = members;
        if (t1_items > p->max_t1_items) p->max_t1_items = t1_items;
    }
    p->blob_bytes = base;
    uint8_t* h = p->header;
    put32(h + 0, kMagic);
    put32(h + 4, kVersion);
    put32(h + 8, (uint32_t)p->dims.d_out);
    put32(h + 12, p->d_pad);
    put32(h + 16, (uint32_t)E);
    put32(h + 20, (uint32_t)p->dims.rank);
    put64(h + 24, p->blob_bytes);
    put64(h + 32, kHeaderBytes);
    put64(h + 40, p->header_bytes);
    return BITSMOE_OK;
}

static bitsmoe_plan* new_plan(const bitsmoe_dims* d) {
    bitsmoe_plan* p = (bitsmoe_plan*)calloc(1, sizeof(bitsmoe_plan));
    if (!p) return nullptr;
    p->dims = *d;
    p->counts = (uint32_t*)calloc(8 * (size_t)d->n_experts, sizeof(uint32_t));
    if (!p->counts) {
        free(p);
        return nullptr;
    }
    return p;
}

}  // namespace bitsmoe

using namespace bitsmoe;

BITSMOE_API int bitsmoe_pack_plan(const bitsmoe_dims* dims, const uint8_t* widths_host, bitsmoe_plan** out) {
    if (!out) return BITSMOE_EINVAL;
    *out = nullptr;
    if (!dims_ok(dims) || !widths_host) return BITSMOE_EINVAL;
    const int E = dims->n_experts, r = dims->rank;
    for (size_t i = 0; i < (size_t)E * r; i++)
        if (!width_ok(widths_host[i])) return BITSMOE_EWIDTH;
    bitsmoe_plan* p = new_plan(dims);
    if (!p) return BITSMOE_ENOMEM;
    for (int e = 0; e < E; e++) {
        uint32_t* c = p->counts + 8 * (size_t)e;
        for (int k = 0; k < r; k++) {
            int g = group_of_width(widths_host[(size_t)e * r + k]);
            c[g < 0 ? 7 : g]++;
        }
    }
    int rc = finish_plan(p);
    if (rc) {
        bitsmoe_plan_free(p);
        return rc;
    }
    *out = p;
    return BITSMOE_OK;
}

BITSMOE_API int bitsmoe_plan_from_header(const void* header_host, uint64_t n_bytes, int32_t d_in, int32_t top_k,
                                         bitsmoe_plan** out) {
    if (!out) return BITSMOE_EINVAL;
    *out = nullptr;
    if (!header_host) return BITSMOE_EINVAL;
    const uint8_t* h = (const uint8_t*)header_host;
    if (n_bytes < kHeaderBytes) return BITSMOE_ESIZE;
    if (get32(h) != kMagic || get32(h + 4) != kVersion) return BITSMOE_EFORMAT;
    bitsmoe_dims d;
    d.d_in = d_in;
    d.top_k = top_k;
    d.d_out = (int32_t)get32(h + 8);
    d.n_experts = (int32_t)get32(h + 16);
    d.rank = (int32_t)get32(h + 20);
    if (get32(h + 8) > (1u << 30) || get32(h + 16) > (1u << 20) || get32(h + 20) > 65535u) return BITSMOE_EFORMAT;
    if (d_in < 1 || top_k < 1 || top_k > 1024) return BITSMOE_EINVAL;
    if (!dims_ok(&d)) return BITSMOE_EFORMAT;
    uint64_t hb = kHeaderBytes + kDirEntryBytes * (uint64_t)d.n_experts;
    if (n_bytes < hb) return BITSMOE_ESIZE;
    bitsmoe_plan* p = new_plan(&d);
    if (!p) return BITSMOE_ENOMEM;
    for (int e = 0; e < d.n_experts; e++) {
        const uint8_t* dir = h + kHeaderBytes + kDirEntryBytes * (uint64_t)e;
        uint32_t total = 0;
        for (int g = 0; g < 8; g++) {
            p->counts[8 * (size_t)e + g] = get16(dir + 44 + 2 * g);
            total += get16(dir + 44 + 2 * g);
        }
        if (total != (uint32_t)d.rank) {
            bitsmoe_plan_free(p);
            return BITSMOE_EFORMAT;
        }
    }
    int rc = finish_plan(p);
    // the rebuilt header must equal the given one byte for byte
    if (!rc && memcmp(p->header, h, hb) != 0) rc = BITSMOE_EFORMAT;
    if (rc) {
        bitsmoe_plan_free(p);
        return rc;
    }
    *out = p;
    return BITSMOE_OK;
}

BITSMOE_API void bitsmoe_plan_free(bitsmoe_plan* plan) {
    if (!plan) return;
    free(plan->header);
    free(plan->counts);
    free(plan);
}

BITSMOE_API uint64_t bitsmoe_plan_blob_bytes(const bitsmoe_plan* plan) { return plan ? plan->blob_bytes : 0; }

BITSMOE_API uint64_t bitsmoe_plan_header_bytes(const bitsmoe_plan* plan) { return plan ? plan->header_bytes : 0; }

BITSMOE_API int bitsmoe_plan_get_dims(const bitsmoe_plan* plan, bitsmoe_dims* out) {
    if (!plan || !out) return BITSMOE_EINVAL;
    *out = plan->dims;
    return BITSMOE_OK;
}

BITSMOE_API int bitsmoe_plan_write_header(const bitsmoe_plan* plan, void* host_out, uint64_t capacity) {
    if (!plan || !host_out) return BITSMOE_EINVAL;
    if (capacity < plan->header_bytes) return BITSMOE_ESIZE;
    memcpy(host_out, plan->header, plan->header_bytes);
    return BITSMOE_OK;
}

BITSMOE_API int bitsmoe_read_status(const int32_t* status_dev, void* stream, int32_t* out_host) {
    if (!status_dev || !out_host) return BITSMOE_EINVAL;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(out_host, status_dev, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return set_cuda_error(e);
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return set_cuda_error(e);
    return BITSMOE_OK;
}

BITSMOE_API const char* bitsmoe_strerror(int code) {
    switch (code) {
        case BITSMOE_OK: return "ok";
        case BITSMOE_EINVAL: return "invalid argument (dimension, NULL or misaligned pointer)";
        case BITSMOE_EWIDTH: return "width outside {0,1,2,3,4,6,8,16}";
        case BITSMOE_ESIZE: return "buffer smaller than required";
        case BITSMOE_ECUDA: return g_cuda_msg;
        case BITSMOE_EFORMAT: return "blob header or directory does not parse";
        case BITSMOE_ENOMEM: return "host allocation failed";
        default: return "unknown error code";
    }
}

BITSMOE_API int bitsmoe_version(void) { return 100; }
