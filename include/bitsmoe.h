/*
 * bitsmoe.h -- C ABI of the B200 (sm_100a) library for the decode-time hot
 * path of BitsMoE's spectral MoE gate/up projection.
 *
 * The method (BitsMoE study-note page, "BitsMoE: Cost-Aware Bit Allocation In
 * spectral Space for MoE LLM Quantization"):
 *   - Methodology, first split: one projection's experts share an input basis
 *     Phi (from an SVD of the stacked expert matrices), so W_e x = P_e (Phi^T x)
 *     and z = Phi^T x is computed once per token and reused by every selected
 *     expert.
 *   - second split: W_e = sum_k a_{e,k} p_{e,k} phi_k^T with unit directions
 *     p_{e,k}; a_{e,k} is the component's amplitude.
 *   - Usage: each component is stored at a width b in {0,1,2,3,4,6,8,16};
 *     0 drops it, 16 keeps it as fp16.
 *   - Execution: components of equal width are grouped and packed by bit plane.
 * Quantiser (not on the pages; mid-rise, one fp16 scale per component):
 *   s = fp16(2 max|p| / (2^b - 1)),  q = clamp(floor(p / s + 2^(b-1)), 0, 2^b - 1),
 *   w = s (q - (2^b - 1)/2).
 * Forward, per routed (token t, slot j) with expert e = ids[t][j]:
 *   Y_e[t][j][i] = sum_b [ sum_bit 2^bit sum_{k in G_b} c_k bit_{k,bit,i}
 *                          - (2^b - 1)/2 sum_{k in G_b} c_k ]  (+ fp16 group),
 *   c_k = a_{e,k} s_{e,k} z_{t,k};  Y_sum[t][i] = sum_j g[t][j] Y_e[t][j][i].
 *
 * Conventions for every call:
 *   - Pointers marked "dev" are device pointers (cudaMalloc, torch tensors...),
 *     "host" are host pointers.  The caller allocates and owns every buffer,
 *     and the library never allocates device memory.  The one piece of device
 *     state it keeps is the fixed scratch array of
 *     bitsmoe_layer_forward_t1_noalloc (static device memory of the loaded
 *     library, used by that call only).  Plans are host objects the library
 *     allocates and bitsmoe_plan_free frees.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every device
 *     call is asynchronous on that stream; only bitsmoe_read_status waits.
 *   - Return 0 on success or a negative BITSMOE_E* code.  Argument errors are
 *     found on the host before any launch.  Data errors found on the device
 *     (non-finite component, bad scale, expert id out of range, ...) are OR-ed
 *     into a caller-owned device int32 `status` word as BITSMOE_ST_* bits; the
 *     affected outputs are zero; nothing traps.
 *   - fp16 values are passed as uint16_t bit patterns; fp32 as float.
 *   - All arrays are dense, row-major, with the shapes written beside them.
 *
 * Packed format v2 (the blob written by bitsmoe_pack; little-endian).  Blob =
 * header (64 B) | directory (E x 64 B) | expert 0 | expert 1 | ... ;
 * d_pad = roundup(d_out, 32).
 *   header: u32 magic "BMOE" | u32 version 2 | u32 d_out | u32 d_pad | u32 E |
 *           u32 r | u64 total bytes | u64 64 | u64 64+64E | 16 zero bytes.
 *   directory entry e: u64 base (byte offset of expert e) | u64 bytes |
 *           u32 group offset from base [7] | u16 count [8] | u32 0;
 *           groups and counts in width order 16,8,6,4,3,2,1 (count[7] = width 0).
 *   group b in {1,2,3,4,6,8}, n members in ascending k, np = roundup(n,32):
 *           u16 idx[np] | u16 fp16 scale[np] | f32 amp[np] |
 *           u32 planes[b][np/32][d_pad]: bit m of word [j][w][i] is bit j of
 *           q for member 32w+m at row i (rows fastest: a warp reads one plane
 *           word of 32 rows as 128 contiguous bytes, and consecutive plane
 *           words of one group, all rows, are one contiguous block).
 *   group 16, np = roundup(n,8): u16 idx[np] | f32 amp[np] | u16 w16[np][d_pad].
 *   Every padding byte (members >= n, rows >= d_out) is zero.
 */
#ifndef BITSMOE_H
#define BITSMOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ---- */
#define BITSMOE_OK 0
#define BITSMOE_EINVAL (-1)  /* bad dimension, NULL or misaligned pointer */
#define BITSMOE_EWIDTH (-2)  /* a width outside {0,1,2,3,4,6,8,16} */
#define BITSMOE_ESIZE (-3)   /* a buffer smaller than required */
#define BITSMOE_ECUDA (-4)   /* a CUDA launch or API error (text in bitsmoe_strerror) */
#define BITSMOE_EFORMAT (-5) /* a blob header/directory that does not parse */
#define BITSMOE_ENOMEM (-6)  /* host allocation of a plan failed */

/* ---- device status bits ---- */
#define BITSMOE_ST_NONFINITE 1   /* a non-finite component element (its q or w16 is 0) */
#define BITSMOE_ST_BADSCALE 2    /* a scale that is negative, NaN or Inf (its q are 0) */
#define BITSMOE_ST_BADEXPERT 4   /* a routed expert id outside [0, E): zero Y_e row, left out of Y_sum */
#define BITSMOE_ST_TIMEOUT 8     /* a bounded device wait gave up; outputs of that call are invalid */
#define BITSMOE_ST_PLANMISMATCH 16 /* device widths disagree with the plan's widths */
#define BITSMOE_ST_BOUNDS 32       /* bounds-checked build only: a computed index fell outside its
                                      buffer; that access was skipped (outputs of the call invalid) */
#define BITSMOE_ST_NOCONVERGE 64   /* bitsmoe_ssd_decompose: the eigensolver did not converge (or met a
                                      non-finite value); the outputs of the call are invalid */

typedef struct {
    int32_t d_in;      /* input width of the projection (rows of Phi) */
    int32_t d_out;     /* output width (rows of each W_e), >= 1 */
    int32_t n_experts; /* E >= 1 */
    int32_t rank;      /* r = number of spectral components, 1 <= r <= 65535 */
    int32_t top_k;     /* experts per token, >= 1 */
} bitsmoe_dims;

typedef struct bitsmoe_plan bitsmoe_plan;

/* Plan the packed layout of one projection from its widths.
 * widths_host [E][r] uint8 in {0,1,2,3,4,6,8,16}.  On success *out holds a
 * new plan (free it with bitsmoe_plan_free).  Errors: EINVAL (dims, NULL),
 * EWIDTH, ENOMEM.  (Usage: the width set; Execution: grouping by width.) */
int bitsmoe_pack_plan(const bitsmoe_dims *dims, const uint8_t *widths_host, bitsmoe_plan **out);

/* Rebuild a plan from the first bitsmoe_plan_header_bytes() bytes of a saved
 * blob (host copy) plus the two dims a blob does not store (d_in, top_k).
 * Checks magic, version and every directory entry.  Errors: EINVAL, EFORMAT,
 * ESIZE (n_bytes shorter than header + directory), ENOMEM. */
int bitsmoe_plan_from_header(const void *header_host, uint64_t n_bytes, int32_t d_in, int32_t top_k,
                             bitsmoe_plan **out);

void bitsmoe_plan_free(bitsmoe_plan *plan);

/* Total bytes of the blob (header + directory + all experts); 0 for NULL. */
uint64_t bitsmoe_plan_blob_bytes(const bitsmoe_plan *plan);

/* Bytes of header + directory (= 64 + 64 E); 0 for NULL. */
uint64_t bitsmoe_plan_header_bytes(const bitsmoe_plan *plan);

/* Copies the plan's dims to *out.  Errors: EINVAL. */
int bitsmoe_plan_get_dims(const bitsmoe_plan *plan, bitsmoe_dims *out);

/* Copies header + directory (bitsmoe_plan_header_bytes bytes) to host_out.
 * Errors: EINVAL, ESIZE. */
int bitsmoe_plan_write_header(const bitsmoe_plan *plan, void *host_out, uint64_t capacity);

/* Per-component fp16 scale s = fp16(2 max_i |p_i| / (2^b - 1)) for widths
 * 1..8 (IEEE fp32 divide, round-to-nearest-even to fp16); 0 for widths 0 and
 * 16.  comps dev [E][r][d_out] f32, widths dev [E][r] u8 (same values as the
 * plan's), scales dev [E][r] u16 (out).  A component with a non-finite element
 * gets scale 0 and BITSMOE_ST_NONFINITE.  status dev int32 or NULL.
 * Errors: EINVAL, ECUDA. */
int bitsmoe_compute_scales(const bitsmoe_plan *plan, const float *comps, const uint8_t *widths,
                           uint16_t *scales, int32_t *status, void *stream);

/* Quantise and pack one projection into `blob` (dev, bitsmoe_plan_blob_bytes
 * bytes, 16-byte aligned).  comps dev [E][r][d_out] f32 (unit directions
 * p_{e,k}), widths dev [E][r] u8, scales dev [E][r] u16 (fp16 bits, from
 * bitsmoe_compute_scales or the caller's own), amps dev [E][r] f32.  Every
 * byte of the blob is written; the result is bit-exact with the format above.
 * Data errors go to *status (dev int32 or NULL).  Errors: EINVAL, ECUDA.
 * (Execution: grouping by width, bit-plane packing; Usage: 0 and 16.) */
int bitsmoe_pack(const bitsmoe_plan *plan, const float *comps, const uint8_t *widths,
                 const uint16_t *scales, const float *amps, void *blob, int32_t *status, void *stream);

/* Test support: unpack every component of `blob` (dev) to q dev [E][r][d_out]
 * u16 (the b-bit integer for widths 1..8, the raw fp16 bits for width 16, 0
 * for width 0).  Errors: EINVAL, ECUDA. */
int bitsmoe_unpack_q(const bitsmoe_plan *plan, const void *blob, uint16_t *q, void *stream);

/* Shared projection Z[t][k] = sum_i PhiT[k][i] X[t][i] (first split: z =
 * Phi^T x, once per token).  phi_t dev [r][d_in] fp16 (row k = phi_k),
 * X dev [T][d_in] fp16, Z dev [T][r] f32 (out); fp32 accumulation.
 * phi_t and X must be 16-byte aligned and d_in a multiple of 8.  T = 0 is a
 * no-op.  Errors: EINVAL, ECUDA. */
int bitsmoe_shared_proj(const uint16_t *phi_t, const uint16_t *X, float *Z, int32_t T, int32_t d_in,
                        int32_t r, void *stream);

/* Workspace bytes bitsmoe_expert_forward needs for T tokens. */
uint64_t bitsmoe_expert_workspace_bytes(const bitsmoe_plan *plan, int32_t T);

/* Routed expert forward of one projection from a packed blob.
 *   blob dev (packed by bitsmoe_pack for `plan`), Z dev [T][r] f32,
 *   topk_ids dev [T][top_k] int32, gate_w dev [T][top_k] f32 (applied as
 *   given, not renormalised), Y_experts dev [T][top_k][d_out] f32 or NULL,
 *   Y_sum dev [T][d_out] f32, workspace dev (>= bitsmoe_expert_workspace_bytes,
 *   256-byte aligned; contents need no initialisation), status dev or NULL.
 * Tokens that share an expert are grouped so each expert's planes are read
 * once per call.  Errors: EINVAL, ESIZE, ECUDA. */
int bitsmoe_expert_forward(const bitsmoe_plan *plan, const void *blob, const float *Z, const int32_t *topk_ids,
                           const float *gate_w, int32_t T, float *Y_experts, float *Y_sum, void *workspace,
                           uint64_t workspace_bytes, int32_t *status, void *stream);

/* One projection's buffers for bitsmoe_layer_forward. */
typedef struct {
    const bitsmoe_plan *plan; /* host plan of `blob` */
    const void *blob;         /* dev packed blob */
    const uint16_t *phi_t;    /* dev [r][d_in] fp16 */
    float *Z;                 /* dev [T][r] f32 out, or NULL (then kept in the workspace) */
    float *Y_experts;         /* dev [T][top_k][d_out] f32 out, or NULL */
    float *Y_sum;             /* dev [T][d_out] f32 out */
} bitsmoe_proj_io;

/* Workspace bytes bitsmoe_layer_forward needs for T tokens. */
uint64_t bitsmoe_layer_workspace_bytes(const bitsmoe_plan *gate, const bitsmoe_plan *up, int32_t T);

/* Number of kernels one bitsmoe_layer_forward call launches for T tokens with
 * these plans: 1 when the fused single-token path applies (T = 1 and the
 * shapes fit one CTA per SM), else 7 (routing groups, then per projection the
 * shared projection, the experts and the routed combine); 0 for T = 0.
 * Errors: EINVAL. */
int bitsmoe_layer_launches(const bitsmoe_plan *gate, const bitsmoe_plan *up, int32_t T);

/* Gate and up projections of one spectral MoE layer for T tokens: z = Phi^T x
 * for both projections, then the routed experts of both, then their routed
 * sums.  X dev [T][d_in] fp16; topk_ids / gate_w as in bitsmoe_expert_forward
 * (shared by both projections).  The two plans must agree on d_in and top_k.
 * workspace dev (>= bitsmoe_layer_workspace_bytes, 256-byte aligned) must be
 * zero-filled, all of it, once before its first use: its head holds the fused
 * single-token path's state -- a launch counter and the z rows, each tagged
 * with the launch that wrote it -- which every call (a timed-out one too)
 * leaves ready for the next.  If it is ever cleared again, clear all of it:
 * restarting the counter while z rows of earlier calls keep their tags could
 * let a call take a stale row.  Calls that share a workspace must not overlap
 * on the GPU.  With T = 1 the fused kernel adds the CTAs' partial rows with
 * fp32 atomic additions, whose order, and so the last bits of Y_sum and
 * Y_experts, can differ between runs; with T > 1 the routed sum is formed in
 * slot order.  Errors: EINVAL, ESIZE, ECUDA. */
int bitsmoe_layer_forward(const bitsmoe_proj_io *gate, const bitsmoe_proj_io *up, const uint16_t *X,
                          const int32_t *topk_ids, const float *gate_w, int32_t T, void *workspace,
                          uint64_t workspace_bytes, int32_t *status, void *stream);

/* bitsmoe_layer_forward for a decode loop that knows the layer it runs next.
 * The BitsMoE pages have no counterpart to this call: at one token the shared
 * projections' Phi^T are most of the bytes a layer reads, and they are
 * weights, known before the next layer's input exists.  So while this call
 * evaluates its experts (when HBM would otherwise be idle) the fused
 * single-token path prefetches next_phi_t_gate and next_phi_t_up -- the next
 * layer's Phi^T, dev [r][d_in] fp16 each, the same shape as this layer's --
 * into L2, and the next call reads them from there.  The bytes still come
 * from HBM once per layer; only their time moves.  Other paths (T > 1, or
 * shapes the fused path does not take) ignore the two pointers.
 *   Arguments as in bitsmoe_layer_forward, plus next_phi_t_gate / next_phi_t_up:
 *   both NULL (no prefetch, the same as bitsmoe_layer_forward) or both
 *   16-byte aligned device pointers; nothing is written through them.
 * Errors: those of bitsmoe_layer_forward; EINVAL when only one is NULL or one
 * is misaligned. */
int bitsmoe_layer_forward_chained(const bitsmoe_proj_io *gate, const bitsmoe_proj_io *up, const uint16_t *X,
                                  const int32_t *topk_ids, const float *gate_w, int32_t T, void *workspace,
                                  uint64_t workspace_bytes, const uint16_t *next_phi_t_gate,
                                  const uint16_t *next_phi_t_up, int32_t *status, void *stream);

/* Single-token layer forward (T = 1) that allocates nothing: the same fused
 * kernel as bitsmoe_layer_forward, with its scratch taken from one fixed 1 MiB
 * array that the library keeps in device memory (every GPU that loads the
 * library holds it until the process exits).  The BitsMoE pages have no
 * counterpart to this call; it exists for callers that cannot allocate device
 * memory or hand out a workspace -- a serving runtime that owns all device
 * memory through its own pool, a plugin that is only given its input and
 * output buffers, or a decode loop that must not call cudaMalloc because it
 * synchronises the device and cannot be recorded into a CUDA graph.
 *   gate, up, X, topk_ids, gate_w, status: as in bitsmoe_layer_forward with
 *   T = 1 (topk_ids / gate_w hold one row of top_k entries).
 * The first call on each device looks up the array's device address; make
 * that first call before any stream capture.  The array starts zeroed and
 * every call leaves it ready for the next, so calls that overlap on the GPU
 * (two streams, two host threads) race and must be serialised by the caller.
 * Errors: EINVAL (dims, NULL or misaligned pointers), ESIZE (shapes the
 * single-launch kernel cannot hold, or scratch beyond 1 MiB), ECUDA. */
int bitsmoe_layer_forward_t1_noalloc(const bitsmoe_proj_io *gate, const bitsmoe_proj_io *up, const uint16_t *X,
                                     const int32_t *topk_ids, const float *gate_w, int32_t *status, void *stream);

/* ---- the expert FFN after the gate and up projections ----
 * The BitsMoE pages decompose an expert's gate and up projections and stop
 * there.  These calls finish the expert the usual gated way, with a dense fp16
 * down projection per expert (the pages leave it uncompressed):
 *   h[t][j][m] = SiLU(Yg[t][j][m]) * Yu[t][j][m],   SiLU(v) = v / (1 + e^-v),
 *   out[t][i]  = sum_j g[t][j] sum_m Wd[e][i][m] h[t][j][m],   e = topk_ids[t][j],
 * where Yg, Yu are the Y_experts outputs of the gate and up projections. */
typedef struct {
    int32_t d_model;   /* rows of each down matrix: the layer's hidden width (the gate/up d_in), >= 1 */
    int32_t d_ff;      /* columns: the gate/up projections' d_out; a multiple of 8 */
    int32_t n_experts; /* E >= 1 */
    int32_t top_k;     /* experts per token, >= 1 */
} bitsmoe_ffn_dims;

/* Workspace bytes bitsmoe_ffn_down needs for T tokens (0 when the single-token
 * kernel applies: T <= 1 and top_k x d_ff fp32 fit one CTA's shared memory). */
uint64_t bitsmoe_ffn_down_workspace_bytes(const bitsmoe_ffn_dims *dims, int32_t T);

/* Kernels one bitsmoe_ffn_down call launches: 1 on the single-token path, else 3
 * (routing groups, the experts' rows, the slot-order sum); 0 for T = 0.
 * Errors: EINVAL. */
int bitsmoe_ffn_down_launches(const bitsmoe_ffn_dims *dims, int32_t T);

/* SiLU(gate) * up and the down projection of the routed experts, summed per token.
 *   w_down dev [E][d_model][d_ff] fp16 (16-byte aligned), Y_gate / Y_up dev
 *   [T][top_k][d_ff] f32 (16-byte aligned), topk_ids dev [T][top_k] int32,
 *   gate_w dev [T][top_k] f32 (applied as given), out dev [T][d_model] f32,
 *   workspace dev (>= bitsmoe_ffn_down_workspace_bytes, 256-byte aligned, no
 *   initialisation needed; may be NULL when that size is 0), status dev or NULL.
 * A slot whose id is outside [0, E) contributes nothing and sets
 * BITSMOE_ST_BADEXPERT.  fp32 arithmetic; each token's sum runs in slot order, so
 * results do not depend on timing.  The single-token kernel is launched with
 * programmatic dependent launch: it requests its weight rows into L2 before it
 * waits for the kernel ahead of it in the stream (the layer call that wrote
 * Y_gate / Y_up), and reads nothing else before that wait.
 * Errors: EINVAL (dims, NULL or misaligned pointers), ESIZE (workspace), ECUDA. */
int bitsmoe_ffn_down(const bitsmoe_ffn_dims *dims, const uint16_t *w_down, const float *Y_gate, const float *Y_up,
                     const int32_t *topk_ids, const float *gate_w, int32_t T, float *out, void *workspace,
                     uint64_t workspace_bytes, int32_t *status, void *stream);

/* Workspace bytes bitsmoe_ffn_forward needs for T tokens: the layer's, then the
 * down step's (each on a 256-byte boundary). */
uint64_t bitsmoe_ffn_workspace_bytes(const bitsmoe_plan *gate, const bitsmoe_plan *up, int32_t T);

/* Kernels one bitsmoe_ffn_forward call launches for T tokens: those of
 * bitsmoe_layer_forward plus those of bitsmoe_ffn_down.  Errors: EINVAL. */
int bitsmoe_ffn_launches(const bitsmoe_plan *gate, const bitsmoe_plan *up, int32_t T);

/* The whole expert FFN of one layer for T tokens: bitsmoe_layer_forward, then
 * bitsmoe_ffn_down on the two projections' per-slot outputs.
 *   gate, up: as in bitsmoe_layer_forward, with Y_experts set in both (16-byte
 *   aligned; they are the down step's inputs); the plans agree on d_out.
 *   w_down dev [E][d_in][d_out] fp16, 16-byte aligned (d_model = the plans' d_in,
 *   d_ff = their d_out, a multiple of 8).  X, topk_ids, gate_w: as in
 *   bitsmoe_layer_forward.  out dev [T][d_in] f32.
 *   workspace dev (>= bitsmoe_ffn_workspace_bytes, 256-byte aligned): its head is
 *   the layer's workspace, with the same rules (zero-filled once before first use,
 *   calls that share it must not overlap); the down step's part follows it.
 * On one token the down kernel follows the fused layer kernel by programmatic
 * dependent launch (see bitsmoe_ffn_down).  Errors: those of the two calls. */
int bitsmoe_ffn_forward(const bitsmoe_proj_io *gate, const bitsmoe_proj_io *up, const uint16_t *w_down,
                        const uint16_t *X, const int32_t *topk_ids, const float *gate_w, int32_t T, float *out,
                        void *workspace, uint64_t workspace_bytes, int32_t *status, void *stream);

/* ---- the offline step before the decode path: decomposition and widths ----
 * Shared-basis spectral decomposition of one projection's experts (study-note page,
 * Methodology: first split, W_cat = U S Phi^T over the experts stacked vertically,
 * (E d_out) x d_in, Phi the shared input basis, P = U S = W_cat Phi; second split,
 * a_{e,k} = ||P_e[:,k]||, p_{e,k} = P_e[:,k] / a_{e,k}, so that
 * W_e = sum_k a_{e,k} p_{e,k} phi_k^T).  The right singular vectors and the
 * singular values are taken as the eigenvectors and the square roots of the
 * eigenvalues of the Gram matrix W_cat^T W_cat (fp32 GEMMs in cuBLAS without TF32,
 * the fp32 symmetric eigensolver of cuSOLVER; both loaded on first use); the r
 * largest are kept, in descending order, each phi_k with the sign that makes its
 * entry of largest magnitude positive.  The outputs are the inputs of
 * bitsmoe_compute_scales / bitsmoe_pack and of the decode path.  Needs a GPU. */

/* Workspace bytes of bitsmoe_ssd_decompose (0 for bad dims, or when cuBLAS or
 * cuSOLVER cannot be loaded or no device is usable). */
uint64_t bitsmoe_ssd_workspace_bytes(int32_t n_experts, int32_t d_out, int32_t d_in, int32_t rank);

/*   W dev [E][d_out][d_in] f32 (the expert matrices), 1 <= rank <= d_in;
 *   phi_t dev [rank][d_in] fp16 (out: row k = phi_k), phi_t32 dev [rank][d_in] f32
 *   (out: the same in fp32) or NULL, sigma dev [rank] f32 (out: the singular
 *   values) or NULL, amps dev [E][rank] f32 (out), comps dev
 *   [E][rank][d_out] f32 (out: unit p_{e,k}; 0 where a = 0), workspace dev
 *   (>= bitsmoe_ssd_workspace_bytes, 256-byte aligned), status dev or NULL
 *   (BITSMOE_ST_NOCONVERGE).  Errors: EINVAL, ESIZE, ECUDA (also when cuBLAS or
 *   cuSOLVER cannot be loaded). */
int bitsmoe_ssd_decompose(const float *W, int32_t n_experts, int32_t d_out, int32_t d_in, int32_t rank,
                          uint16_t *phi_t, float *phi_t32, float *sigma, float *amps, float *comps, void *workspace,
                          uint64_t workspace_bytes, int32_t *status, void *stream);

/* Widths by descending amplitude within each expert, ties to the lower k (the
 * study-note page, Usage, gives the width set; this call takes the allocation's
 * counts): per expert the counts[0] components of largest a get
 * widths_in_order[0], the next counts[1] get widths_in_order[1], and so on.
 *   amps_host [E][r] f32, widths_in_order [n] in {0,1,2,3,4,6,8,16}, counts [n]
 *   summing to r, widths_host [E][r] u8 (out).  Host only.
 * Errors: EINVAL (NULL, counts that do not sum to r), EWIDTH. */
int bitsmoe_assign_widths(const float *amps_host, int32_t n_experts, int32_t rank, const uint8_t *widths_in_order,
                          const int32_t *counts, int32_t n, uint8_t *widths_host);

/* ---- the allocation of widths (offline, host) ----
 * The study-note page, Methodology, third split: activation-dependent importance
 * beta_{e,k} = sum over calibration (token, slot) pairs routed to e of
 * g (phi_k^T x)^2, importance a_{e,k}^2 beta_{e,k}, cost L_{e,k}(b) =
 * a^2 beta eps_{e,k,b}; Usage: widths in {0,1,2,3,4,6,8,16} chosen jointly under a
 * bit budget (a component of d_out elements costs d_out b bits).  The pages leave
 * eps undefined: eps_{e,k,b} = ||p_{e,k} - stored p_{e,k}||^2 at width b with this
 * library's quantiser (0 bits: ||p||^2; 16 bits: fp16(p)).  All host, fp64, in a
 * fixed order (results independent of the thread count).  Width index order of
 * eps arrays: 0,1,2,3,4,6,8,16. */

/* comps_host [E][r][d_out] f32 -> eps_host [E][r][8] f64 (NaN at
 * every width for a component with a non-finite element).  Errors: EINVAL. */
int bitsmoe_fqcm_eps(const float *comps_host, int32_t n_experts, int32_t rank, int32_t d_out, double *eps_host);

/* beta_host [E][r] f64 from Z_host [T][r] f32 (z = Phi^T x of T calibration tokens,
 * e.g. from bitsmoe_shared_proj), topk_ids_host [T][top_k], gate_w_host [T][top_k];
 * ids outside [0, E) are skipped.  Errors: EINVAL. */
int bitsmoe_fqcm_beta(const float *Z_host, const int32_t *topk_ids_host, const float *gate_w_host, int32_t T,
                      int32_t top_k, int32_t n_experts, int32_t rank, double *beta_host);

/* widths_host [E][r] u8 minimising sum L_{e,k}(b) under sum d_out b <= budget_bits,
 * through the linear relaxation of this multiple-choice knapsack: per component the
 * lower convex hull of its (bits, loss) points from width 0, then all hull segments
 * in order of loss saved per bit (ties: lower e r + k, then earlier segment), taken
 * while they fit, the first that does not fit ending the allocation (at budgets
 * where the relaxation is integral this is the integer optimum).  A component
 * whose cost is not finite keeps width 0.  loss_host (out, total cost) or NULL.
 * amps_host [E][r] f32, beta_host [E][r] f64, eps_host [E][r][8] f64.
 * Errors: EINVAL. */
int bitsmoe_allocate_widths(const float *amps_host, const double *beta_host, const double *eps_host,
                            int32_t n_experts, int32_t rank, int32_t d_out, uint64_t budget_bits,
                            uint8_t *widths_host, double *loss_host);

/* Waits for `stream`, then copies the device status word to *out_host.
 * Errors: EINVAL, ECUDA. */
int bitsmoe_read_status(const int32_t *status_dev, void *stream, int32_t *out_host);

/* Static text for a return code (for ECUDA, the last CUDA error seen by this
 * thread's last failing call). */
const char *bitsmoe_strerror(int code);

/* Library version: 100 * major + minor. */
int bitsmoe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* BITSMOE_H */
