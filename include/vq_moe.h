/*
 * vq_moe.h -- C ABI of the VQ-MoE expert-path library (libvqmoe.so).
 *
 * The library computes the hot path of vector-quantised (VQ) MoE checkpoints
 * on one NVIDIA B200 (sm_100a): expert weights are stored as packed
 * log2(K)-bit indices into a per-module codebook of K fp16 centroids of
 * d weights each, with one fp16 scale per (row, 64 weights), and dead
 * "skipzero" rows dropped. The kernels reconstruct the weights on the fly and
 * contract them with the activations of the tokens routed to each expert.
 *
 * Format (VQ model cards):
 *   - Qwen3.5-397B-A17B-VQ-2.6bpw card, "Methodology": one index per
 *     d-weight subvector into a per-tensor fp16 codebook, fp16 scale per
 *     (row, 64 weights).
 *   - Qwen3.5-397B-A17B-VQ-2.4bpw card, "Methodology": codes packed into
 *     uint32 words, row-local, 32-code blocks. The bit order inside a block
 *     is not printed; this library reads it as: code j of a row occupies
 *     bits [j*b, j*b+b) of the row's bit string, bit i of the string being
 *     bit (i % 32) of word i / 32 (least significant bit first).
 *   - same card, "Changelog 2026-10-01 (vq-skipzero)": dead output rows
 *     carry no codes or scales and output exact zeros.
 *
 * Conventions for every call:
 *   - Pointers marked "device" are CUDA device pointers the caller owns; the
 *     library never allocates, frees or retains them after the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Device calls are asynchronous on that stream and never
 *     synchronise the host; their results are valid once the stream has run.
 *   - The return value reports argument errors and launch failures
 *     synchronously. Nothing is launched when a call returns an error.
 *   - fp16 and bf16 values are passed as their uint16 bit patterns.
 */
#ifndef VQ_MOE_H
#define VQ_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum vq_status {
    VQ_OK = 0,
    VQ_ERR_ARG = 1,           /* NULL where a pointer is required, bad size or shape */
    VQ_ERR_ALIGN = 2,         /* a pointer is not aligned as documented */
    VQ_ERR_UNSUPPORTED = 3,   /* geometry (d, bits) or size the kernels do not implement */
    VQ_ERR_WORKSPACE = 4,     /* workspace NULL, misaligned or smaller than required */
    VQ_ERR_CUDA = 5,          /* a CUDA runtime call or kernel launch failed */
    VQ_ERR_DEVICE_CHECK = 6   /* a kernel recorded an error: it gave up a bounded wait, or
                                 vq_fit met an index out of range (see vq_moe_check) */
} vq_status;

/* Output element types. */
enum { VQ_F32 = 0, VQ_BF16 = 1 };

/*
 * One VQ module: the weights of one (layer, projection) for E experts that
 * share one codebook (reading of "per-tensor codebook": one codebook per
 * projection of a layer, shared by all of that layer's experts).
 *
 * Expert e's weight matrix is W_e [rows, cols] with
 *   W_e[r, c] = fp32(codebook[code_e(r, c / d)][c % d]) * fp32(scale_e[r, c / 64])
 *               (+ fp32(bias_e[r, c / 64]) for a module with biases)
 * where code_e(r, j) is the j-th b-bit code of row r. The bias is the
 * optional affine arm: the cards' fallback format "affine 3-bit, group 64"
 * (Qwen3.5-397B-A17B-VQ-2.4bpw card, Changelog 2026-09-20) is stated without
 * its formula; this library reads it as the group-wise affine form
 * w = s * q + b with an fp16 scale and an fp16 bias per (row, 64 weights),
 * which is d = 1 with the codebook C[q] = q plus the bias.
 *
 * Requirements: d in {1, 2, 4, 8}; cols a multiple of 64 and of 32*d (whole
 * 32-code blocks and whole scale groups); (d, bits) one of the implemented
 * geometries (vq_geometry_supported).
 */
typedef struct vq_module {
    int32_t E;        /* experts */
    int32_t rows;     /* output features of each expert */
    int32_t cols;     /* input features of each expert */
    int32_t d;        /* weights per code (subvector length) */
    int32_t bits;     /* code width b; the codebook has K = 2^bits entries */
    /* device, 16-byte aligned: packed codes of the live rows, expert-major,
     * live rows of one expert in increasing row order; each row is
     * vq_packed_words(1, cols / d, bits) uint32 words. */
    const uint32_t *codes;
    /* device, 2-byte aligned: fp16 scales [live rows, cols / 64], same row order. */
    const uint16_t *scales;
    /* device, 16-byte aligned: fp16 codebook [2^bits, d]. */
    const uint16_t *codebook;
    /* device or NULL: live-row bitmap [E, ceil(rows / 32)]; bit (r % 32) of
     * word r / 32 is 1 when row r of the expert is live. NULL: every row of
     * every expert is live and expert e's row r is packed row e*rows + r. */
    const uint32_t *live_bitmap;
    /* device, required when live_bitmap is set: [E, ceil(rows / 32)], the
     * packed-row index of the first live row at or after row 32*w of expert
     * e (vq_live_rank builds it). */
    const uint32_t *live_rank;
    /* number of packed rows in `codes` and `scales` (the extent the kernels
     * may read); required when live_bitmap is set, ignored (E * rows)
     * otherwise. */
    int64_t live_rows;
    /* device, 2-byte aligned, or NULL (no bias): fp16 biases [live rows,
     * cols / 64], the same layout as `scales`. */
    const uint16_t *biases;
} vq_module;

/* A SwiGLU MoE layer: y = sum_j w_j * down_e( silu(gate_e x) * up_e x ).
 * gate and up: rows = inter, cols = hidden; down: rows = hidden, cols = inter;
 * all three with the same E. Each has its own codebook and geometry. */
typedef struct vq_moe_layer {
    vq_module gate;
    vq_module up;
    vq_module down;
} vq_moe_layer;

/* Human-readable name of a status. Never NULL. */
const char *vq_status_str(vq_status s);

/* 1 when the kernels implement geometry (d, bits), else 0. */
int vq_geometry_supported(int32_t d, int32_t bits);

/* ------------------------------------------------------------ host packing */

/* uint32 words of `rows` packed rows of `ncode` codes of `bits` bits:
 * rows * (ncode / 32) * bits (a 32-code block is exactly `bits` words).
 * Returns 0 when ncode is not a positive multiple of 32 or bits not in 1..16. */
size_t vq_packed_words(int64_t rows, int32_t ncode, int32_t bits);

/* Host. Packs codes [E, rows, ncode] (uint16, values < 2^bits) into the
 * row-local LSB-first layout, keeping only live rows when live_bitmap (host,
 * [E, ceil(rows/32)]) is given (skipzero: live rows are byte-identical to a
 * full packing). out: host, out_words >= vq_packed_words(live rows, ncode,
 * bits). *rows_written receives the number of packed rows.
 * Errors: VQ_ERR_ARG (NULL, bad sizes, a code >= 2^bits, out too small). */
vq_status vq_pack(const uint16_t *codes, int32_t E, int32_t rows, int32_t ncode, int32_t bits,
                  const uint32_t *live_bitmap, uint32_t *out, size_t out_words, size_t *rows_written);

/* Host. Keeps the live rows of per-row fp16 scales [E, rows, ngroups]
 * (ngroups = cols / 64) in the same order as vq_pack. */
vq_status vq_pack_scales(const uint16_t *scales, int32_t E, int32_t rows, int32_t ngroups,
                         const uint32_t *live_bitmap, uint16_t *out, size_t out_elems,
                         size_t *rows_written);

/* Host. Builds live_rank [E, ceil(rows/32)] from a live bitmap (both host).
 * Bits at or beyond `rows` in the last word of an expert must be 0. */
vq_status vq_live_rank(const uint32_t *live_bitmap, int32_t E, int32_t rows, uint32_t *rank_out);

/* ------------------------------------------------------------ device calls */

/* Diagnostic. codes_out: device uint16 [rows, cols/d]: the codes of expert
 * `expert`'s rows; dead rows are filled with 0xFFFF. */
vq_status vq_unpack(const vq_module *m, int32_t expert, uint16_t *codes_out, void *stream);

/* Diagnostic. w_out: device fp32 [rows, cols]: the dequantised weights of
 * `expert` (exact: the fp16 x fp16 product is exact in fp32); dead rows +0. */
vq_status vq_dequant(const vq_module *m, int32_t expert, float *w_out, void *stream);

/* y[t, r] = sum_c W_expert[r, c] * x[t, c] for t < T, accumulated in fp32.
 * x: device bf16 [T, cols], 16-byte aligned. y: device [T, rows] of y_dtype
 * (VQ_F32 or VQ_BF16, round to nearest even). Dead rows give +0.
 * The contraction runs on tensor cores (the decode GEMV) with the codebook
 * entries and the activations in fp16. Every 64-column group of a token's
 * activations is multiplied by a power of two 2^k that puts its largest |x|
 * in [2^14, 2^15) before the fp16 rounding, so any finite bf16 input keeps
 * fp16's full precision (down to 2^-28 of the group's largest value) and
 * nothing overflows; the group's fp32 partial sum is multiplied by its fp32
 * scale and by 2^-k (exact). Results are accurate wherever y is a normal fp32
 * number. */
vq_status vq_gemv(const vq_module *m, int32_t expert, const uint16_t *x, int32_t T, void *y,
                  int32_t y_dtype, void *stream);

/* Bytes of workspace vq_gemm needs for T tokens of module m's shape; 0 on
 * invalid arguments. */
size_t vq_gemm_workspace_size(const vq_module *m, int32_t T);

/* The prefill path's tcgen05 GEMM for one expert (a dense building block with
 * the same arithmetic as vq_moe_prefill's expert GEMMs): for t < T,
 *   y0[t, r] = sum_c W0_expert[r, c] * x[t, c]     (module m0)
 *   y1[t, r] = sum_c W1_expert[r, c] * x[t, c]     (module m1, when not NULL)
 * m1, when given, must have m0's E, rows, cols, d and bits: the two share
 * each weight-tile pass, as a layer's gate and up projections do. The weight
 * tiles are decoded on chip to fp16 (fp16(centroid) x fp16(group scale),
 * rounded to nearest even) and contracted with the tokens' activations in
 * fp16 on the tensor cores, accumulated in fp32. Each token's activations are
 * multiplied by 2^k (largest |x| in [2^14, 2^15)) before their fp16 rounding
 * and the fp32 result by 2^-k. x: device bf16 [T, cols], 16-byte aligned.
 * y0, y1: device fp32 [T, rows], 16-byte aligned. workspace: device,
 * 256-byte aligned, vq_gemm_workspace_size(m0, T) bytes (its first word is the
 * error word that vq_moe_check reads). Requirements as vq_moe_prefill's for
 * each module (VQ_ERR_UNSUPPORTED otherwise). Errors: VQ_ERR_ARG (bad sizes,
 * expert out of range, m1 of another shape), VQ_ERR_ALIGN, VQ_ERR_WORKSPACE. */
vq_status vq_gemm(const vq_module *m0, const vq_module *m1, int32_t expert, const uint16_t *x, int32_t T,
                  float *y0, float *y1, void *workspace, size_t ws_bytes, void *stream);

/* Top-k routing and expert bucketing of T tokens: the MoE router of the VQ
 * model cards' layers (Qwen3.8-Flash-Next-VQ-4.4bpw card: 10 of 512 experts
 * per token; gemma-4-26b-a4b-it-VQ-6.2bpw card: 128 experts, top 8). The
 * cards print no tie or normalisation rule; the readings taken here follow.
 * logits: device fp32 [T, E]. Per token the top_k experts are taken in order
 * of larger logit first, ties to the smaller expert index, NaN last.
 * weights: renorm != 0 -> softmax over the selected logits; renorm == 0 ->
 * the full softmax over all E experts, evaluated at the selected ones.
 * Outputs (device): ids int32 [T, top_k]; weights fp32 [T, top_k];
 * offsets int32 [E + 1] (exclusive prefix sums of per-expert pair counts);
 * perm int32 [T * top_k]: pair indices p = t*top_k + j grouped by expert,
 * increasing p inside each expert's bucket.
 * Requires 1 <= top_k <= min(E, 32), E <= 4096, T * top_k < 2^31. */
vq_status vq_route(const float *logits, int32_t T, int32_t E, int32_t top_k, int32_t renorm,
                   int32_t *ids, float *weights, int32_t *offsets, int32_t *perm, void *stream);

/* Which MoE path a workspace is sized for. */
enum { VQ_MODE_DECODE = 0, VQ_MODE_PREFILL = 1 };

/* Bytes of workspace vq_moe_decode (mode VQ_MODE_DECODE) or vq_moe_prefill
 * (VQ_MODE_PREFILL) need for T tokens and top_k. 0 on invalid arguments. */
size_t vq_moe_workspace_size(const vq_moe_layer *L, int32_t T, int32_t top_k, int32_t mode);

/* MoE SwiGLU layer for decode-sized batches (a few tokens per expert). T = 0
 * launches nothing and returns VQ_OK; x, logits and y may then be NULL:
 *   y[t] = sum_j w[t, j] * W_down,e_j ( silu(W_gate,e_j x[t]) * (W_up,e_j x[t]) )
 * with (e_j, w[t, j]) from vq_route on `logits` (device fp32 [T, E]).
 * Range: the tensor cores take 16-bit fp16 operands, so each token's
 * activation row, and each (token, expert) row of the SwiGLU output h, is
 * multiplied by a power of two that puts its largest magnitude in
 * [2^14, 2^15) before its fp16 rounding; the fp32 results are multiplied back
 * exactly. Any finite bf16 input is therefore taken at fp16's full precision
 * (down to 2^-28 of its row's largest value) without overflow; g, u, h and y
 * are fp32, and results are accurate wherever those are normal fp32 numbers.
 * x: device bf16 [T, hidden], 16-byte aligned. y: device [T, hidden] of
 * y_dtype, 16-byte aligned. workspace: device, 256-byte aligned, at least
 * vq_moe_workspace_size(L, T, top_k, VQ_MODE_DECODE) bytes; it holds the
 * routing tables and the intermediate activations and may be reused by the
 * next call once this one has run. Sums over experts run in slot order j,
 * so results are deterministic. */
vq_status vq_moe_decode(const vq_moe_layer *L, const uint16_t *x, int32_t T, const float *logits,
                        int32_t top_k, int32_t renorm, void *y, int32_t y_dtype, void *workspace,
                        size_t ws_bytes, void *stream);

/* The same layer for prefill-sized batches (many tokens per expert): per
 * expert bucket a grouped GEMM on the tcgen05 tensor cores with the weight
 * tiles decoded on chip to fp16 (fp16(centroid) x fp16(group scale), rounded
 * to nearest even). Same arguments, result definition and range handling as
 * vq_moe_decode; workspace sized with VQ_MODE_PREFILL. Additionally requires,
 * for every module, a packed row that is a multiple of 16 bytes
 * ((cols / d / 32) * bits divisible by 4) and cols a multiple of 64 * CH,
 * CH being the smallest number of 64-column steps whose codes fill a whole
 * number of 16-byte units (VQ_ERR_UNSUPPORTED otherwise). */
vq_status vq_moe_prefill(const vq_moe_layer *L, const uint16_t *x, int32_t T, const float *logits,
                         int32_t top_k, int32_t renorm, void *y, int32_t y_dtype, void *workspace,
                         size_t ws_bytes, void *stream);

/* Prefill of a long prompt in chunks, so that scratch memory is bounded by
 * the chunk rather than the prompt (the Qwen3.8-Flash-Next-VQ-4.4bpw card
 * chunks its speculative prefill in 2048 tokens, and the GLM-5.3-Flash-VQ-2.7bpw
 * card tells serving loops to chunk the prefill at 2048). Tokens [c0, c0 + chunk) of x and logits
 * go through vq_moe_prefill into rows [c0, c0 + chunk) of y, one chunk after
 * another on `stream`; the last chunk takes the remaining tokens. Each
 * token's output depends only on its own x row and logits, so the result is
 * vq_moe_prefill's over all T tokens. The workspace is sized for one chunk:
 * vq_moe_workspace_size(L, min(T, chunk), top_k, VQ_MODE_PREFILL) bytes, and
 * is reused by every chunk. chunk < 1 returns VQ_ERR_ARG; other errors as
 * vq_moe_prefill (a chunk that fails stops the loop; earlier chunks stay
 * queued). */
vq_status vq_moe_prefill_chunked(const vq_moe_layer *L, const uint16_t *x, int32_t T, const float *logits,
                                 int32_t top_k, int32_t renorm, int32_t chunk, void *y, int32_t y_dtype,
                                 void *workspace, size_t ws_bytes, void *stream);

/* ---- Data-free VQ fit: the step that makes a module's codebook, codes and
 * scales from a bf16 weight tensor ----
 * The VQ model cards ("Methodology" of Qwen3.5-397B-A17B-VQ-2.6bpw,
 * Qwen3.8-Flash-Next-VQ-4.4bpw, GLM-5.3-Flash-VQ-2.7bpw) fit each tensor's codebook
 * in pure weight space: k-means / Lloyd over the weight subvectors of a drawn
 * subsample, no Hessian, activation statistics or calibration data; an fp16
 * scale per (row, 64 weights). For one tensor W (bf16, row-major
 * [rows, cols]; subvector i = row i / (cols/d), weights d*(i % (cols/d)) ..)
 * vq_fit computes:
 *   scales   fp16 [rows, cols/64]: the group's largest |w| (the cards give the
 *            scale's shape only; this is the reading taken),
 *   v        = w / scale per subvector, fp32 (0 where the scale is 0),
 *   `iters`  Lloyd steps over the subvectors sample[0..n_sample) from the
 *            centroids v[init[k]]: each point goes to its nearest centroid
 *            (fp32 squared distance, components summed in order with no fused
 *            multiply-add, ties to the lower index); a centroid with points
 *            becomes their exact mean rounded to fp32, one with none keeps its
 *            value,
 *   codebook fp16 [K, d]: the final centroids rounded to fp16,
 *   codes    uint16 [rows, cols/d]: every subvector's nearest codebook entry.
 * Pack codes with vq_pack for the expert path. All arrays are device memory;
 * sample and init hold subvector indices drawn by the caller. Requirements:
 * d in {1, 2, 4, 8}; cols a multiple of 64; 2 <= K <= 65536 and K*d <= 32768
 * (the centroids sit in shared memory); K <= n_sample <= 2^22; iters >= 0;
 * rows*cols/d < 2^31 (VQ_ERR_ARG otherwise); w, scales, codebook and codes
 * 16-byte aligned (VQ_ERR_ALIGN). An index outside [0, rows*cols/d) is
 * skipped and sets the workspace's error word (see vq_moe_check). Results are
 * deterministic: centroid sums are exact integers. Workspace:
 * vq_fit_workspace_size(K, d) bytes (0 for invalid K or d), 256-byte aligned,
 * owned by the caller. Asynchronous on `stream`. */
size_t vq_fit_workspace_size(int32_t K, int32_t d);
vq_status vq_fit(const uint16_t *w, int32_t rows, int32_t cols, int32_t d, int32_t K, const int32_t *sample,
                 int32_t n_sample, const int32_t *init, int32_t iters, uint16_t *scales, uint16_t *codebook,
                 uint16_t *codes, void *workspace, size_t ws_bytes, void *stream);

/* Diagnostic (synchronises `stream`). Every wait of the library's pipelined
 * kernels on an on-chip barrier is bounded; a kernel that gives up records a
 * nonzero word at offset 0 of the MoE workspace it ran with (the routing
 * kernel of each vq_moe_decode / vq_moe_prefill call clears it) and stops
 * without completing its outputs. vq_fit records the same word in its own
 * workspace for a sample or init index out of range (each call clears it). Returns VQ_ERR_DEVICE_CHECK when the word
 * of `workspace` is set after the work queued on `stream`, VQ_OK when not,
 * VQ_ERR_WORKSPACE for a NULL or misaligned workspace. */
vq_status vq_moe_check(const void *workspace, void *stream);

/* vq_moe_decode without a workspace argument, for callers that cannot
 * allocate device memory: code running inside a host framework that owns
 * every device allocation and allows no new ones on its serving path, or a
 * program that reaches this library through a thin C FFI without a CUDA
 * memory API. The paper has no counterpart; the layer computed is exactly
 * vq_moe_decode's, with the same arguments minus the workspace.
 *
 * Scratch: one 16 MiB file-scope device array inside the library. Every GPU
 * that loads the library holds it until the process exits. Calls whose
 * vq_moe_workspace_size(L, T, top_k, VQ_MODE_DECODE) exceeds 16 MiB return
 * VQ_ERR_WORKSPACE and launch nothing.
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture. The address is kept per device and looked up
 * again when the calling thread's context is not the one it was found in
 * (for instance after cudaDeviceReset).
 * Sharing: all calls on a device use the same array and it keeps the last
 * call's contents (no call needs it zeroed: each writes what it reads).
 * Calls that overlap on the GPU (other streams, other host threads) race on
 * it; serialise them. The library allocates nothing for this call. */
vq_status vq_moe_decode_noalloc(const vq_moe_layer *L, const uint16_t *x, int32_t T, const float *logits,
                                int32_t top_k, int32_t renorm, void *y, int32_t y_dtype, void *stream);

/* Bound on the polls of every barrier wait in the pipelined kernels that the
 * calling thread launches from now on (no counterpart on the pages; a
 * failure-detection hook). polls < 0 restores the default, 2^22 polls (each
 * may suspend the waiting thread briefly); 0 makes every wait give up at
 * once. A wait that gives up makes its CTA stop: it lets
 * the copies and tensor-core operations it issued complete, frees its tensor
 * memory, records a nonzero word in the workspace (see vq_moe_check) and
 * returns without completing its outputs. Nothing faults or hangs. Errors:
 * VQ_ERR_ARG when polls > 2^32 - 1. */
vq_status vq_set_wait_limit(int64_t polls);

/* Tracing (no counterpart on the pages; an observability hook for timing
 * each kernel stage with the caller's CUDA events). events: host array of
 * n_events cudaEvent_t handles (as void*) created by the caller, or NULL to
 * switch tracing off. While set, the calling thread's vq_moe_decode and
 * vq_moe_prefill record events[i] on their stream at stage boundary i:
 *   decode:  0 | route | 1 | gate/up GEMV | 2 | SwiGLU | 3 | down GEMV | 4 | combine | 5
 *   prefill: 0 | route | 1 | gather | 2 | gate/up GEMM | 3 | h scales + down GEMM | 4 | combine | 5
 * Boundaries beyond n_events are not recorded. The library does not own
 * the events. Errors: VQ_ERR_ARG when n_events < 0. */
vq_status vq_set_trace_events(void *const *events, int32_t n_events);

#ifdef __cplusplus
}
#endif

#endif /* VQ_MOE_H */
