/*
 * moe_grouped.h — C ABI of the B200 (sm_100a) MoE expert-MLP hot path.
 *
 * The path: top-k router softmax -> stable permutation of tokens into expert-contiguous
 * rows with per-expert counts (split_sizes) -> grouped GEMM fc1 (gate|up) with the
 * ScaledSwiGLU epilogue (SiLU(gate) * up * routing probability) -> grouped GEMM fc2 ->
 * unpermute and combine of the k expert outputs of every token; plus the backward
 * dgrad/wgrad grouped GEMMs, and an MXFP8 variant (E4M3 values, one E8M0 scale per 32
 * consecutive values along K).
 *
 * Pages: "Efficient MoE training for biological foundation models" — sitech.ge,
 * sections "Grouped experts instead of a Python loop" and "Reducing memory and
 * quantisation cost"; news.bpdata.com, sections 1) to 3).
 *
 * Conventions shared by every call:
 *   - All pointers are DEVICE pointers unless stated otherwise; the caller allocates and
 *     owns every buffer. The library never allocates device memory in these calls.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Every call only enqueues work on it and returns; nothing synchronises the host.
 *   - bf16 tensors are passed as uint16_t* (raw bfloat16 bits); all tensors are dense
 *     row-major with the logical shapes given below.
 *   - The grouped GEMMs read and write their operands and outputs with TMA and 16-byte
 *     vector accesses: those buffers start on 16-byte boundaries (a misaligned one is
 *     an argument error, MOE_ERR_INVALID_ARG).
 *   - Return value: a moe_status_t. Argument errors are reported synchronously before
 *     anything is launched. Errors found by kernels (bad expert index, split sizes that
 *     do not add up, a wait that ran out of time) set a device error word that
 *     moe_device_status() reads. CUDA launch errors return MOE_ERR_CUDA.
 *   - Sizes: T tokens, E experts (1..1024), k experts per token (1..min(E,32)),
 *     H hidden size, F expert FFN size, R = T*k routed rows.
 */
#ifndef MOE_GROUPED_H
#define MOE_GROUPED_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, negative size, k > E, workspace too small */
  MOE_ERR_UNSUPPORTED = 2,   /* valid but unsupported shape (e.g. H % 256 != 0) */
  MOE_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
  MOE_ERR_DEVICE_CHECK = 4,  /* a kernel detected bad data (see moe_device_status) */
  MOE_ERR_TIMEOUT = 5        /* a kernel wait exceeded its time budget */
} moe_status_t;

typedef enum { MOE_BF16 = 0, MOE_MXFP8 = 1, MOE_FP8 = 2 } moe_precision_t;

/* Flag OR-ed into grouped_mlp_fwd's `precision`: write yp as fp32 [R, H] instead of bf16
 * (the fc2 accumulator without the bf16 storage rounding). */
#define MOE_OUT_F32 0x100

/* Human-readable name of a status code (static string). */
MOE_API const char* moe_status_string(int status);

/* Synchronises `stream`, then reads and clears the device error word.
 * Returns MOE_OK, MOE_ERR_DEVICE_CHECK, MOE_ERR_TIMEOUT or MOE_ERR_CUDA. */
MOE_API int moe_device_status(void* stream);

/* Number of kernels this library has launched in this process (all devices). */
MOE_API uint64_t moe_launch_count(void);

/*
 * moe_test_stall_gemm — test hook for the timeout path; the pages have no counterpart.
 * Arms a one-shot stall: the grouped GEMM launches of this process (from grouped_mlp_fwd
 * and grouped_mlp_bwd, in launch order) let `skip` launches through, and in the next one
 * the TMA producers issue no copies and every wait gets a budget of timeout_ns
 * (1e5 .. 1e10 ns) instead of 4 s. The first wait for data then runs out: the kernel sets
 * MOE_ERR_TIMEOUT in the device error word, its other roles see the abort or run out in
 * turn, every CTA frees its tensor memory and the launch returns; the context stays
 * usable and later calls run normally. The stalled call's outputs are undefined.
 * Launch order: grouped_mlp_fwd = fc1, fc2; grouped_mlp_bwd = fc2 dgrad, fc2 wgrad,
 * fc1 dgrad, fc1 wgrad.
 */
MOE_API int moe_test_stall_gemm(int skip, uint64_t timeout_ns);

/*
 * moe_route — top-k router softmax.
 * Pages: sitech.ge introduction and news.bpdata.com "dense vs MoE": every token is sent
 * to a few experts whose outputs are weighted by routing weights.
 * Computes, per token t, the softmax of logits[t, :] over all E experts (fp32), selects
 * the k largest logits (equal logits: lower expert index first) in descending order and
 * writes their experts and probabilities; with renorm != 0 the k probabilities are
 * divided by their sum.
 *   logits [T, E] fp32 (input); idx [T, k] int32 (output); prob [T, k] fp32 (output).
 */
MOE_API int moe_route(const float* logits, int T, int E, int k, int renorm, int32_t* idx, float* prob, void* stream);

/*
 * moe_route_bwd — gradient of the router's probabilities with respect to its logits.
 * Pages: sitech.ge introduction (each token's expert outputs are weighted by its routing
 * weights, so the router learns through those weights).
 * The forward (moe_route) is s = softmax(logits) over all E experts, q_j = s[idx_j], and
 * p_j = q_j / sum_m q_m with renorm (else p_j = q_j). Given dprob = dL/dp, writes
 * dlogits = dL/dlogits by the chain rule through those steps:
 *   renorm != 0: dlogits[b] = sum over slots j with idx_j == b of p_j (dprob_j - D),
 *                D = sum_m dprob_m p_m; experts that no slot chose get 0 (logits unused);
 *   renorm == 0: dlogits[b] = s_b (ds_b - sum_c ds_c s_c), ds_b = sum of dprob_j over the
 *                slots j with idx_j == b; s recomputed from logits in fp32.
 *   logits [T, E] fp32 (input; may be NULL with renorm); idx [T, k] int32 and
 *   prob [T, k] fp32 (the forward's outputs); dprob [T, k] fp32 (input);
 *   dlogits [T, E] fp32 (output, every entry written).
 * An index outside [0, E) sets MOE_ERR_DEVICE_CHECK in the device error word and that
 * slot contributes nothing.
 */
MOE_API int moe_route_bwd(const float* logits, const int32_t* idx, const float* prob, const float* dprob, int T,
                          int E, int k, int renorm, float* dlogits, void* stream);

/* Bytes of device scratch moe_permute and moe_route_permute need (per-block expert
 * histograms, and a counter for the fused call). */
MOE_API size_t moe_permute_workspace_size(int T, int k, int E);

/*
 * moe_route_permute — moe_route followed by moe_permute, with the routing, the per-block
 * expert histogram and its scan in one kernel launch (three launches instead of five).
 * Same pages as the two calls. Same arguments and outputs, bit for bit, as
 *   moe_route(logits, T, E, k, renorm, idx, prob) then
 *   moe_permute(x, idx, prob, T, H, E, k, precision, xp, xp_scale, row_map, probs_perm,
 *               split_sizes, offsets, workspace, workspace_bytes);
 * here idx and prob are outputs and both are required. The fused launch covers k that
 * divides 1024 and E <= 256; other shapes run the two calls' kernels. workspace: at least
 * moe_permute_workspace_size(T, k, E) bytes (its last 256 bytes hold a counter that the
 * call zeroes itself). Calls that share a workspace must not overlap on the GPU.
 */
MOE_API int moe_route_permute(const float* logits, const uint16_t* x, int T, int H, int E, int k, int renorm,
                              int precision, int32_t* idx, float* prob, void* xp, uint8_t* xp_scale,
                              int32_t* row_map, float* probs_perm, int32_t* split_sizes, int32_t* offsets,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_permute — stable permutation of the T*k routed slots into expert-contiguous rows.
 * Pages: sitech.ge "Grouped experts instead of a Python loop" and news.bpdata.com
 * section 1): tokens are grouped per expert and the grouped GEMM receives the per-expert
 * token counts (split_sizes); NeMo AutoModel page, Transformers v5 back-ends: grouped_mm
 * runs on tokens sorted by expert.
 * Slot s = t*k + j (token t, choice j). Within an expert, rows keep ascending slot order.
 *   x [T, H] bf16 (input); idx [T, k] int32 (input, values in [0, E));
 *   prob [T, k] fp32 (input, may be NULL when probs_perm is NULL);
 *   precision MOE_BF16: xp [R, H] bf16, xp_scale ignored (may be NULL);
 *   precision MOE_MXFP8: xp [R, H] E4M3 codes (uint8), xp_scale [R, H/32] E8M0 codes,
 *     each row quantised along H in blocks of 32 (H % 32 == 0);
 *   row_map [R] int32 (output): row of slot s in xp;
 *   probs_perm [R] fp32 (output, may be NULL): probs_perm[row_map[s]] = prob[s];
 *   split_sizes [E] int32 (output); offsets [E+1] int32 (output, exclusive prefix sum);
 *   workspace: device scratch of at least moe_permute_workspace_size(T, k, E) bytes.
 * Requires H % 8 == 0 (bf16) or H % 32 == 0 (MXFP8). An index outside [0, E) sets
 * MOE_ERR_DEVICE_CHECK in the device error word and its slot gets row_map = -1.
 */
MOE_API int moe_permute(const uint16_t* x, const int32_t* idx, const float* prob, int T, int H, int E, int k,
                int precision, void* xp, uint8_t* xp_scale, int32_t* row_map, float* probs_perm,
                int32_t* split_sizes, int32_t* offsets, void* workspace, size_t workspace_bytes, void* stream);

/* Largest per-block histogram table moe_permute_noalloc can hold, in int32 entries:
 * ceil(T*k / 1024) * E must not exceed it (e.g. T*k <= 2,097,152 with E = 128). */
#define MOE_PERMUTE_NOALLOC_MAX_COUNTS 262144

/*
 * moe_permute_noalloc — moe_permute for callers that cannot allocate device memory.
 * The pages have no counterpart to this call; it is the same stable permutation as
 * moe_permute (same arguments, same outputs, bit for bit) minus the workspace argument.
 *
 * Who needs it: hosts that must not allocate once they are running — an inference
 * server or embedded runtime that plans all device memory at start-up and forbids
 * cudaMalloc afterwards (it can fail under memory pressure and it synchronises the
 * device), or a plain C caller with no caching allocator that would otherwise pay a
 * cudaMalloc/cudaFree pair around every call. The caller still allocates and passes all
 * inputs and outputs; only the scratch table is provided by the library.
 *
 * Scratch: a fixed table of MOE_PERMUTE_NOALLOC_MAX_COUNTS int32 (1 MiB) in static
 * device memory that every GPU which loads the library holds until the process exits.
 * Sizes that need more return MOE_ERR_UNSUPPORTED (with a message on stderr) before
 * anything is launched. This call never calls cudaMalloc, cudaFree or any allocating
 * routine. The first call on each device looks up the table's device address (with that
 * device current); make that first call before any stream capture. All calls share the
 * one table and it keeps the last call's contents (every entry a call reads is written
 * by the same call first), so calls whose GPU work overlaps — on two streams, or from
 * two host threads — race on it and must be serialised by the caller. The looked-up
 * address is kept for the life of the process: do not call this after cudaDeviceReset on
 * that device (the table would be at a new address in the new context).
 */
MOE_API int moe_permute_noalloc(const uint16_t* x, const int32_t* idx, const float* prob, int T, int H, int E, int k,
                                int precision, void* xp, uint8_t* xp_scale, int32_t* row_map, float* probs_perm,
                                int32_t* split_sizes, int32_t* offsets, void* stream);

/* Bytes of device scratch moe_permute_capacity needs. */
MOE_API size_t moe_permute_capacity_workspace_size(int T, int k, int E);

/*
 * moe_permute_capacity — the capacity-padded dispatch of the padded "batched_mm" expert
 * back-end (NeMo AutoModel page, Transformers v5 features: experts_implementation in
 * {eager, batched_mm, grouped_mm}), as a comparison point for the dropless grouped path.
 * Every expert gets exactly C rows: the first min(n_e, C) of its slots in slot order
 * s = t*k + j (the stable order of moe_permute) fill rows [e*C, e*C + n_e), the rest of
 * its C rows are zeros, and its slots past C are dropped (row_map[s] = -1; moe_unpermute
 * and moe_gather_slots skip them, so a dropped slot contributes nothing).
 *   x, idx, prob as moe_permute; C >= 0 the capacity (e.g. ceil(factor * T*k / E));
 *   xp [E*C, H] bf16 (MOE_BF16) or E4M3 codes with xp_scale [E*C, H/32] (MOE_MXFP8);
 *   row_map [R] int32 (slot -> padded row or -1); probs_perm [E*C] fp32 or NULL (zero on
 *   padded rows); split_sizes [E] (= C each) and offsets [E+1] (= e*C) for
 *   grouped_mlp_fwd on the padded rows; kept [E] int32 or NULL: min(n_e, C).
 *   workspace: moe_permute_capacity_workspace_size(T, k, E) bytes.
 */
MOE_API int moe_permute_capacity(const uint16_t* x, const int32_t* idx, const float* prob, int T, int H, int E, int k,
                                 int C, int precision, void* xp, uint8_t* xp_scale, int32_t* row_map,
                                 float* probs_perm, int32_t* split_sizes, int32_t* offsets, int32_t* kept,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_permute_rows — the data movement of moe_permute alone, for a tensor that follows
 * an existing row_map (e.g. the gradient of the layer output in the backward pass):
 * dst[row_map[t*k + j]] = src[t]. src [T, H] bf16, dst [R, H] bf16, H % 8 == 0.
 */
MOE_API int moe_permute_rows(const uint16_t* src, const int32_t* row_map, int T, int H, int k, uint16_t* dst, void* stream);

/* Bytes of scratch moe_permute_rows_mxfp8 needs: the token of every permuted row. */
MOE_API size_t moe_permute_rows_mxfp8_workspace_size(int T, int k);

/*
 * moe_permute_rows_mxfp8 — moe_permute_rows fused with the MXFP8 quantisation of the
 * permuted rows (news.bpdata.com section 2: one scale per 32 consecutive values along a
 * GEMM's contraction axis) in the two forms the backward GEMMs read, so that the bf16
 * permuted tensor is never written:
 *   rows form (rows_codes, rows_atoms): codes [R, H], blocks of 32 along H, scale atoms
 *     grouped per 128-row expert tile (the layout of grouped_mlp_fwd's xp_scale, and of
 *     moe_mxfp8_bwd_operands.dy_rows);
 *   cols form (cols_codes, cols_atoms): codes [R, H], blocks of 32 rows restarting at every
 *     expert's first row, atoms in mxfp8_quantize_grouped's layout (dy_cols, xp_cols).
 * Row row_map[t*k + j] of both is src[t] (a dropless row_map: R = T*k rows, every row
 * owned by one slot). split_sizes [E] on the device (sum = R). Either output pair may be
 * NULL. Each atom buffer holds mxfp8_grouped_atoms_bytes(E, R, H) bytes and is zeroed
 * first (bytes of rows or blocks past an expert's end stay 0). H % 128 == 0.
 * workspace: moe_permute_rows_mxfp8_workspace_size(T, k) bytes.
 */
MOE_API int moe_permute_rows_mxfp8(const uint16_t* src, const int32_t* row_map, int T, int H, int k,
                                   const int32_t* split_sizes, int E, uint8_t* rows_codes, uint8_t* rows_atoms,
                                   uint8_t* cols_codes, uint8_t* cols_atoms, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * moe_unpermute — combine of the k expert outputs of every token.
 * Pages: sitech.ge "Grouped experts instead of a Python loop": the routing weights are
 * applied inside the GroupedMLP kernel, so the combine adds the k rows with weight 1;
 * pass `prob` to weight them here instead (when the MLP ran without probabilities).
 *   out[t] = sum_{j<k} w_tj * yp[row_map[t*k + j]], w = prob[t, j] or 1 if prob == NULL,
 *   accumulated in fp32 in slot order and rounded once to bf16.
 *   yp [R, H] bf16; row_map [R]; prob [T, k] fp32 or NULL; out [T, H] bf16. H % 8 == 0.
 */
MOE_API int moe_unpermute(const uint16_t* yp, const int32_t* row_map, const float* prob, int T, int H, int k,
                  uint16_t* out, void* stream);

/* Scale layouts of mxfp8_quantize's output. PLAIN is the [rows, K/32] grid. MMA arranges
 * the scales of a K-major matrix [N, K] (N and K multiples of 128) in the 512-byte atoms
 * the block-scaled tensor-core instruction consumes: atom (g, j) holds rows
 * [128 g, 128 g + 128) and K blocks [4 j, 4 j + 4) at byte offset (g * K/128 + j) * 512;
 * inside it, row r's four bytes form the 32-bit word (r % 32) * 4 + r / 32, byte
 * (block % 4). Stacked expert matrices [E, N, K] number their row groups e * N/128 + n/128. */
#define MOE_SCALES_PLAIN 0
#define MOE_SCALES_MMA 1

/*
 * mxfp8_quantize — MXFP8 quantisation of a batch of bf16 matrices in[batch, rows, cols].
 * Pages: news.bpdata.com section 2) and sitech.ge "Reducing memory and quantisation
 * cost": one scale per block of 32 consecutive values; 16-bit masters are quantised
 * every step (section 3).
 * Per block of 32 values with amax = max|v|: scale X = 2^(floor(log2 amax) - 8) stored
 * as E8M0 (exponent clamped to [-127, 127]; amax == 0 gives code 0); elements are
 * v / X rounded to nearest-even E4M3, saturating at +-448.
 *   axis 0: blocks along cols (cols % 32 == 0): codes [batch, rows, cols],
 *           scales [batch, rows, cols/32]; transpose_out must be 0.
 *   axis 1: blocks along rows (rows % 32 == 0).
 *           transpose_out = 1: codes [batch, cols, rows], scales [batch, cols, rows/32]
 *             (the transposed matrix quantised along its rows: K-major weights);
 *           transpose_out = 0: codes [batch, rows, cols], scales [batch, rows/32, cols].
 *   scale_layout: MOE_SCALES_PLAIN, or MOE_SCALES_MMA (axis 1 with transpose_out, or
 *           axis 0 without; rows and cols multiples of 128) for weights handed to the
 *           block-scaled GEMMs.
 */
MOE_API int mxfp8_quantize(const uint16_t* in, int batch, int rows, int cols, int axis, int transpose_out,
                           int scale_layout, uint8_t* codes, uint8_t* scales, void* stream);

/* Bytes of scratch grouped_mlp_fwd needs (the fc1 output `a` when saved == NULL). */
MOE_API size_t grouped_mlp_workspace_size(int E, int R, int H, int F, int precision, int training);

/* Bytes of the buffer grouped_mlp_fwd fills for the backward pass (training mode):
 * h = [gate | up] pre-activations [R, 2F] bf16, then a: [R, F] bf16 (MOE_BF16) or
 * [R, F] E4M3 codes followed by their scale atoms (MOE_MXFP8); each part starts on a
 * 256-byte boundary. */
MOE_API size_t grouped_mlp_saved_size(int E, int R, int H, int F, int precision);

/*
 * grouped_mlp_fwd — fc1 (gate|up) -> ScaledSwiGLU -> fc2 over expert-contiguous rows.
 * Pages: news.bpdata.com section 1) (grouped GEMM with split_sizes, equal to the
 * per-expert loop) and section 3) (GroupedLinear -> ScaledSwiGLU -> GroupedLinear fused
 * into one pattern); sitech.ge "Grouped experts instead of a Python loop" (routing
 * weights applied inside the GroupedMLP kernel).
 * For every expert e with rows [off_e, off_e + split_sizes[e]):
 *   h = xp_e @ w1[e]            (K = H, N = 2F; gate = h[:, :F], up = h[:, F:])
 *   a = SiLU(gate) * up * p     (p = probs_perm of the row, 1 if probs_perm == NULL)
 *   yp_e = a @ w2[e]            (K = F, N = H)
 * MOE_BF16: xp [R, H] bf16, w1 [E, H, 2F] bf16, w2 [E, F, H] bf16; scales ignored;
 *   a is rounded to bf16 before fc2; fp32 accumulation.
 * MOE_MXFP8: xp [R, H] E4M3 + xp_scale [R, H/32] (plain, as moe_permute writes it);
 *   w1 [E, 2F, H] E4M3 and w2 [E, H, F] E4M3 with their scales in the MOE_SCALES_MMA
 *   layout (as produced by mxfp8_quantize(axis=1, transpose_out=1, MOE_SCALES_MMA));
 *   the fc1 epilogue quantises a along F (blocks of 32) and keeps its scales as MMA
 *   atoms whose row groups are the 128-row tiles of each expert (sum over earlier
 *   experts of ceil(n_e/128), then the tile index); requires H % 128 == 0.
 * MOE_FP8 (per-tensor, see fp8_quantize): xp [R, H] E4M3 codes with xp_scale pointing
 *   to ONE fp32 scale (passed as uint8_t*); w1 [E, 2F, H] and w2 [E, H, F] E4M3 codes
 *   (fp8_quantize with transpose_out) with w1_scale / w2_scale pointing to E fp32 scales
 *   (one per expert); the fc1 epilogue stores a in bf16 and keeps max |a|, then a is
 *   quantised with one E4M3 scale for all rows and fc2 runs on those codes; the
 *   products are rescaled by 1 / (s_A s_B) in the epilogues; requires H % 128 == 0.
 * split_sizes [E] int32 on the device (no host synchronisation happens); R = sum.
 * yp [R, H] bf16 output (fp32 when MOE_OUT_F32 is OR-ed into precision).
 * saved: NULL for inference, else a buffer of
 * grouped_mlp_saved_size() bytes that receives h and a for grouped_mlp_bwd.
 * ws: scratch of grouped_mlp_workspace_size() bytes.
 * Requires H % 64 == 0 and F % 128 == 0.
 */
MOE_API int grouped_mlp_fwd(const void* xp, const uint8_t* xp_scale, const int32_t* split_sizes, int E, int R, int H, int F,
                    const void* w1, const uint8_t* w1_scale, const void* w2, const uint8_t* w2_scale,
                    const float* probs_perm, int precision, void* yp, void* saved, void* ws, size_t ws_bytes,
                    void* stream);

/* Bytes of scratch fp8_quantize needs (one max per tensor). */
MOE_API size_t fp8_quantize_workspace_size(int batch);

/*
 * fp8_quantize — per-tensor FP8 with current scaling (news.bpdata.com section 2, "FP8
 * and MXFP8": FP8 keeps one scale per tensor; E4M3 for forward operands, E5M2 for
 * gradients). For each of `batch` tensors in [batch, rows, cols] bf16: s = fmt_max /
 * max |x| in fp32 (448 for E4M3, 57344 for E5M2; s = 1 for an all-zero tensor), and
 * codes = the fp32 product x * s rounded to the format (nearest even, saturating); a
 * code c stands for decode(c) / s.
 *   fmt: 0 = E4M3, 1 = E5M2; transpose_out: codes [batch, cols, rows] (rows, cols
 *   multiples of 32) instead of [batch, rows, cols] (rows * cols a multiple of 8);
 *   codes uint8 (output); scales [batch] fp32 (output);
 *   workspace: fp8_quantize_workspace_size(batch) bytes.
 */
MOE_API int fp8_quantize(const uint16_t* in, int batch, int rows, int cols, int fmt, int transpose_out, uint8_t* codes,
                         float* scales, void* workspace, size_t workspace_bytes, void* stream);

/* Byte offset inside grouped_mlp_fwd's `saved` buffer of one of its parts ((size_t)-1
 * for a part the precision does not have): part 0 = h [R, 2F] bf16 (all precisions);
 * MOE_BF16 part 1 = a [R, F] bf16; MOE_MXFP8 part 1 = a codes along F [R, F], 2 = their
 * scale atoms (row groups = the experts' 128-row tiles), 3 = a codes along the expert's
 * rows [R, F] (the fc2 weight-gradient operand), 4 = their atoms (the layout of
 * mxfp8_quantize_grouped); MOE_FP8 part 1 = a E4M3 codes [R, F], 2 = a's fp32 scale. */
MOE_API size_t grouped_mlp_saved_offset(int E, int R, int H, int F, int precision, int part);

/* Bytes of scratch grouped_mlp_fwd_combine needs: grouped_mlp_fwd's workspace, then an
 * fp32 [T, H] accumulator and the token of every row. */
MOE_API size_t grouped_mlp_fwd_combine_workspace_size(int E, int R, int H, int F, int precision, int training,
                                                      int T);

/*
 * grouped_mlp_fwd_combine — grouped_mlp_fwd with the unpermute/combine fused into fc2's
 * epilogue (a variant: the routing weights are already applied inside the MLP, sitech.ge
 * "Grouped experts instead of a Python loop", so the combine is a plain sum).
 * out[t] = sum_j yp[row_map[t*k + j]] without writing yp: each fc2 output row is added,
 * from its fp32 accumulator, into an fp32 [T, H] accumulator of its token with 16-byte
 * vector atomics; one pass then rounds that to bf16 out [T, H]. Same arguments as
 * grouped_mlp_fwd (no yp, precision without MOE_OUT_F32) plus row_map [R] (moe_permute's)
 * and T, k with R = T*k. Every row is added in fp32 once, so out is the fp32 sum of the
 * k accumulators rounded once: for k = 2 the result does not depend on the order of the
 * adds; for k > 2 it may differ between runs in the last fp32 bits before rounding.
 * workspace: grouped_mlp_fwd_combine_workspace_size(...) bytes.
 */
MOE_API int grouped_mlp_fwd_combine(const void* xp, const uint8_t* xp_scale, const int32_t* split_sizes, int E, int R,
                                   int H, int F, const void* w1, const uint8_t* w1_scale, const void* w2,
                                   const uint8_t* w2_scale, const float* probs_perm, int precision,
                                   const int32_t* row_map, int T, int k, uint16_t* out, void* saved, void* ws,
                                   size_t ws_bytes, void* stream);

/* Bytes of scratch grouped_mlp_bwd needs: MOE_BF16: dh [R, 2F] bf16 and dprob partial
 * sums; MOE_MXFP8: the dprob partial sums and every quantised GEMM operand. */
MOE_API size_t grouped_mlp_bwd_workspace_size(int E, int R, int H, int F, int precision);

/* Byte offset, inside grouped_mlp_bwd's workspace, of one intermediate of the last call
 * (valid after it completes; (size_t)-1 for a part the precision does not have):
 *   MOE_BF16  part 0: dh = [dg | du] [R, 2F] bf16;
 *   MOE_MXFP8 part 8: dh quantised along its 2F columns: codes [R, 2F], then scale atoms
 *             grouped per 128-row expert tile (row group sum_{e'<e} ceil(n_e'/128) + m
 *             for rows [off_e + 128 m, +128); atom j of a group = k-blocks 4j..4j+3,
 *             row r at 32-bit word (r % 32) * 4 + r / 32; rows past the expert: zeros);
 *             part 9: dh quantised along the expert's rows: codes [R, 2F], then atoms in
 *             the layout of mxfp8_quantize_grouped;
 *   MOE_FP8   part 8: dh E5M2 codes [R, 2F], then (256-byte aligned) its fp32 scale. */
MOE_API size_t grouped_mlp_bwd_workspace_offset(int E, int R, int H, int F, int precision, int part);

/*
 * grouped_mlp_bwd — backward of grouped_mlp_fwd (the "counterpart in the backward
 * pass" of sitech.ge "Reducing memory and quantisation cost").
 * For every expert e (a = SiLU(g) * u * p, with g, u from `saved`):
 *   da = dy_e @ w2[e]^T;  dg = da*p*u*SiLU'(g);  du = da*p*SiLU(g);
 *   dprobs_perm = sum_f da*SiLU(g)*u;  dw2[e] = a_e^T @ dy_e;
 *   dxp_e = [dg | du] @ w1[e]^T;  dw1[e] = xp_e^T @ [dg | du].
 * dy_perm [R, H] bf16 (the layer-output gradient permuted with moe_permute_rows);
 * xp [R, H] bf16 (the permuted layer input, bf16 also on the MXFP8 path);
 * w1 [E, H, 2F] bf16; w2 [E, F, H] bf16 (the masters); probs_perm [R] fp32 or NULL;
 * saved: the buffer filled by grouped_mlp_fwd in training mode (same precision).
 * Outputs: dxp [R, H] bf16, dw1 [E, H, 2F] bf16, dw2 [E, F, H] bf16 (experts with no rows
 * get zeros), dprobs_perm [R] fp32 (may be NULL).
 * MOE_FP8: the gradients dy and dh are quantised to E5M2 with one scale each, the forward
 * operands (xp, the saved a codes, the weights, one scale per expert) are E4M3; dh is
 * stored in bf16 by the fc2-dgrad epilogue (with its max) before its quantisation.
 * MOE_MXFP8: all four GEMMs run on MXFP8 operands quantised along their own contraction
 * axis (blocks of 32): dy and dh along columns for the data gradients, and dy, a
 * (from the forward), dh and xp along rows — in 32-row blocks restarting at every
 * expert's first row — for the weight gradients; the weights are re-quantised along
 * their other axis (grouped_mlp_bwd_mxfp8_operands takes operands already quantised). dh is quantised (both ways) by the fc2-dgrad kernel that computes
 * it, from fp32, and never exists at 16 bits; a along rows comes from the forward (its
 * fc1 epilogue quantises a both ways in training). Requires H % 128 == 0 for MOE_MXFP8.
 */
MOE_API int grouped_mlp_bwd(const void* dy_perm, const int32_t* split_sizes, int E, int R, int H, int F,
                            const void* xp, const void* w1, const void* w2, const float* probs_perm, int precision,
                            const void* saved, uint16_t* dxp, uint16_t* dw1, uint16_t* dw2, float* dprobs_perm,
                            void* ws, size_t ws_bytes, void* stream);

/* Operands of the MXFP8 backward that the caller has already quantised, each a pair (E4M3
 * codes, scale atoms). A pair left NULL is quantised by the call from its bf16 source. */
typedef struct moe_mxfp8_bwd_operands {
  /* dy along H, codes [R, H]; atoms grouped per 128-row expert tile (the layout of
   * grouped_mlp_fwd's xp_scale) */
  const uint8_t* dy_rows;
  const uint8_t* dy_rows_atoms;
  /* dy along the expert's rows, codes [R, H]; atoms in mxfp8_quantize_grouped's layout */
  const uint8_t* dy_cols;
  const uint8_t* dy_cols_atoms;
  /* xp along the expert's rows, codes [R, H]; atoms in mxfp8_quantize_grouped's layout */
  const uint8_t* xp_cols;
  const uint8_t* xp_cols_atoms;
  /* w1 along 2F, codes [E, H, 2F]; w2 along H, codes [E, F, H]: mxfp8_quantize_weights'
   * codes_r / atoms_r */
  const uint8_t* w1_rows;
  const uint8_t* w1_rows_atoms;
  const uint8_t* w2_rows;
  const uint8_t* w2_rows_atoms;
} moe_mxfp8_bwd_operands;

/*
 * grouped_mlp_bwd_mxfp8_operands — grouped_mlp_bwd(..., MOE_MXFP8, ...) with some of its
 * operands already quantised (q, see moe_mxfp8_bwd_operands; q may be NULL). dy_perm may
 * be NULL when both of dy's forms are given, xp when xp_cols is, w1 / w2 when their rows
 * forms are. Same results, outputs and workspace as grouped_mlp_bwd with MOE_MXFP8.
 */
MOE_API int grouped_mlp_bwd_mxfp8_operands(const moe_mxfp8_bwd_operands* q, const void* dy_perm,
                                           const int32_t* split_sizes, int E, int R, int H, int F, const void* xp,
                                           const void* w1, const void* w2, const float* probs_perm, const void* saved,
                                           uint16_t* dxp, uint16_t* dw1, uint16_t* dw2, float* dprobs_perm, void* ws,
                                           size_t ws_bytes, void* stream);

/*
 * mxfp8_quantize_weights — both MXFP8 forms of expert weights in one pass over the bf16
 * masters, which a training step re-quantises after every optimizer step (news.bpdata.com
 * section 2: one scale per 32 consecutive values along the contraction axis):
 *   w [batch, rows, cols] bf16 (w1: [E, H, 2F]; w2: [E, F, H]); rows, cols multiples of 128;
 *   codes_t [batch, cols, rows] E4M3, blocks of 32 along `rows` (the forward GEMM's K),
 *     transposed, and atoms_t their scale atoms: the same bytes as mxfp8_quantize(w, batch,
 *     rows, cols, axis 1, transpose_out, MOE_SCALES_MMA);
 *   codes_r [batch, rows, cols] E4M3, blocks of 32 along `cols` (the data-gradient GEMM's
 *     K), and atoms_r their scale atoms: the same bytes as mxfp8_quantize of w viewed as
 *     [batch * rows, cols], axis 0, MOE_SCALES_MMA.
 * Sizes: codes_t, codes_r batch*rows*cols bytes; atoms_t, atoms_r batch*rows*cols/32 bytes.
 */
MOE_API int mxfp8_quantize_weights(const uint16_t* w, int batch, int rows, int cols, uint8_t* codes_t,
                                   uint8_t* atoms_t, uint8_t* codes_r, uint8_t* atoms_r, void* stream);

/*
 * mxfp8_quantize_grouped — MXFP8 quantisation of expert-contiguous rows along the rows:
 * for every column, blocks of 32 consecutive rows that restart at each expert's first row
 * (the last block of an expert covers its remaining rows, as if zero-padded). This is the
 * operand layout of the weight-gradient GEMMs (contraction over an expert's rows).
 *   in [R, C] bf16, C % 128 == 0; split_sizes [E] on the device (sum = R);
 *   codes [R, C] E4M3 (same layout as in);
 *   atoms: scales in the MMA atom layout, numbered per expert: expert e owns
 *     KG_e = ceil(n_e/128) k-groups; the atom of column group cg (128 columns) and k-group
 *     kg sits at byte (kgoff_e * C/128 + cg * KG_e + kg) * 512, kgoff_e = sum of KG over
 *     earlier experts; inside an atom, column c's word is (c % 32) * 4 + (c % 128) / 32
 *     and block j its byte j % 4; bytes of blocks past an expert's end are zero.
 *     Size: mxfp8_grouped_atoms_bytes(E, R, C).
 */
MOE_API int mxfp8_quantize_grouped(const uint16_t* in, int R, int C, const int32_t* split_sizes, int E,
                                   uint8_t* codes, uint8_t* atoms, void* stream);
MOE_API size_t mxfp8_grouped_atoms_bytes(int E, int R, int C);

/*
 * moe_gather_slots — dst[s] = src[row_map[s]] for s < R (fp32): brings per-row values
 * (e.g. dprobs_perm) back to token/slot order [T, k].
 */
MOE_API int moe_gather_slots(const float* src, const int32_t* row_map, int R, float* dst, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_GROUPED_H */
