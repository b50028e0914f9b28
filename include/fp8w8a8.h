/*
 * fp8w8a8.h - C ABI of the B200 (sm_100a) FP8 W8A8 row-wise linear library.
 *
 * The method (pages cited by title and section):
 *   - "Gemma 4 31B-it QAT, FP8 E4M3 W8A8, text only (unofficial)", header
 *     paragraph: every Linear weight is FP8 E4M3 with one float32 scale per
 *     output channel; activations are quantized to FP8 per token at run
 *     time; other tensors stay bf16.
 *   - Same card, "QAT trained the weights onto a 4-bit grid with one scale
 *     per group of 32 values ... this build rounds the QAT weights again".
 *   - "MI300X 上跑 Gemma 4 E2B：fp8 最快，却离原始权重最远", tip
 *     "E4M3 还是 E4M3FNUZ，都能用": E4M3FNUZ (max 240, no negative zero)
 *     checkpoints are converted at load and serve like the E4M3 build.
 *   - Same article, step 3 boot log: the linear runs as a row-wise scaled
 *     FP8 GEMM (RowWiseTorchFP8ScaledMMLinearKernel on the MI300X).
 *
 * Conventions shared by every entry point:
 *   - All pointers are DEVICE pointers of the current CUDA device unless a
 *     parameter says otherwise. The caller allocates and owns every buffer;
 *     the library allocates no device memory. It keeps one device status word
 *     per device (read with fp8_get_device_status) and a cached driver entry
 *     point for tensor-map encoding.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call
 *     is asynchronous on that stream and returns after enqueueing work.
 *   - Row-major layouts. bf16 values are passed as uint16_t bit patterns.
 *     E4M3 / E4M3FNUZ values are uint8_t codes.
 *   - Host-checkable errors (null pointers, sizes, alignment) return a
 *     non-zero fp8_status BEFORE anything is enqueued. Conditions only the
 *     GPU can see (non-finite inputs, FNUZ NaN codes, inexact FNUZ rows, a
 *     wait that timed out) set bits of the device status word; the call
 *     itself still returns FP8_OK, and the affected rows' outputs are
 *     unspecified.
 *   - Shapes are int64_t; all must be >= 0. A zero-sized problem enqueues
 *     nothing and returns FP8_OK.
 *   - When the status word reports FP8_DEV_TIMEOUT, the outputs of every call
 *     enqueued since the word was last read are undefined (a kernel whose
 *     wait gave up still stores its output tile, from whatever its buffers
 *     held).
 *   - Per-device state (kernel attributes, occupancy figures, the address of
 *     the no-allocation scratch array) is set up on the first call on each
 *     device and cached for the life of the process: the library assumes the
 *     device's primary context lives until the process exits. After a
 *     cudaDeviceReset the library must not be called again in that process.
 *
 * Quantization arithmetic (bit-exact contract, the same in every kernel):
 *   per row r of fp32 values v:  amax = max_k |v[k]|,
 *   s[r] = fp32(amax / 448) (IEEE division, round to nearest even),
 *   code[k] = E4M3_RNE_SATFINITE(fp32(v[k] / s[r])) with a zero result always
 *   encoded as +0 (0x00). A row with amax == 0 gets s = 0 and all-zero codes.
 */
#ifndef FP8W8A8_H
#define FP8W8A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fp8_status {
  FP8_OK = 0,
  FP8_ERR_INVALID_ARG = 1, /* null pointer, negative size, ldx < K        */
  FP8_ERR_ALIGNMENT = 2,   /* a pointer or row pitch is not 16-byte aligned */
  FP8_ERR_SHAPE = 3,       /* K not a multiple of 16 (32 for q4_0), or a
                              dimension beyond the library's limits        */
  FP8_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed            */
  FP8_ERR_UNSUPPORTED = 5, /* the current device is not sm_100             */
  FP8_ERR_SCRATCH_LIMIT = 6 /* the problem needs more scratch than the
                               library's fixed scratch array holds            */
} fp8_status;

/* Bits of the device status word. */
#define FP8_DEV_NONFINITE 0x1u /* a row held NaN/Inf (amax not finite)        */
#define FP8_DEV_NAN_CODE 0x2u  /* FNUZ input held code 0x80 (its NaN)          */
#define FP8_DEV_INEXACT 0x4u   /* FNUZ row not exactly representable in E4M3  */
#define FP8_DEV_TIMEOUT 0x8u   /* a bounded in-kernel wait gave up            */
#define FP8_DEV_BAD_INDEX 0x10u /* an expert id outside [0, num_experts)       */

/* Library version: major * 10000 + minor * 100 + patch. */
int fp8_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* fp8_status_string(fp8_status status);

/* Returns 1 when `device` is an sm_100 GPU this library was built for. */
int fp8_device_supported(int device);

/*
 * Reads and clears the current device's status word. Synchronizes the
 * current device first, so every previously enqueued call is covered.
 * `out` is a HOST pointer.
 */
fp8_status fp8_get_device_status(unsigned int* out);

/*
 * fp8_test_set_fault: test hook for the bounded waits (no counterpart on the
 * pages). Sets, for the current device, the limit of every in-kernel wait to
 * `wait_cycles` SM clock cycles (0 restores the default, 2^31 cycles, about
 * 1.1 s at 1965 MHz), and when `drop_step` >= 0 makes CTA 0 of every decode
 * GEMM launch (fp8_rowwise_linear with M <= 128) skip that pipeline step of
 * its K range: no arrive, no copies, so the MMA's wait for it can end only by
 * the limit. The kernel then records FP8_DEV_TIMEOUT, the producer and MMA
 * roles leave their pipelines, the producer waits for its copies in flight,
 * and the kernel returns (its output is undefined). -1 turns the drop off.
 * Synchronizes the device before and after; not for use while other work of
 * this library runs.
 */
fp8_status fp8_test_set_fault(int64_t wait_cycles, int32_t drop_step);

/*
 * fp8_repack_qat: QAT q4_0-grid weights -> per-output-channel E4M3.
 * Source: model card above, "QAT trained the weights onto a 4-bit grid with
 * one scale per group of 32 values"; header paragraph (one float32 scale per
 * output channel).
 *   q4   [N, K/2] uint8: packed int4, element 2j in the low nibble and 2j+1 in
 *        the high nibble, 4-bit two's complement (values -8..7).
 *   d    [N, K/32] float32: one scale per group of 32 values along K.
 *   w8   [N, K] uint8 out: E4M3 codes of w = fp32(d[n, k/32] * q[n, k])
 *        quantized per row with the contract above.
 *   s_ch [N] float32 out: per-output-channel scales.
 * Requires K % 32 == 0; q4, d, w8 16-byte aligned; s_ch 4-byte aligned.
 * Device status: FP8_DEV_NONFINITE when a row's d*q is not finite.
 */
fp8_status fp8_repack_qat(const uint8_t* q4, const float* d, int64_t N, int64_t K,
                          uint8_t* w8, float* s_ch, void* stream);

/*
 * fp8_convert_fnuz: load-time conversion of an E4M3FNUZ-stored weight to the
 * E4M3 format the GEMM consumes. Source: E2B article, tip "E4M3 还是
 * E4M3FNUZ，都能用" (converted at load; FNUZ max 240, no negative zero).
 *   w8_fnuz [N, K] uint8, s_fnuz [N] float32: the FNUZ weight and scales.
 *   w8 [N, K] uint8 out, s_ch [N] float32 out: E4M3 codes and scales with
 *   dec_e4m3(w8) * s_ch == dec_fnuz(w8_fnuz) * s_fnuz for every element.
 * Per row: with no +-240 code (0x7F / 0xFF) and an exactly halvable scale the
 * bytes are copied and the scale halved; otherwise each value is re-encoded
 * in E4M3 at the same scale (round to nearest even), which is exact except
 * for FNUZ codes with exponent field <= 1 and an odd mantissa; such rows set
 * FP8_DEV_INEXACT. Code 0x80 sets FP8_DEV_NAN_CODE; a non-finite scale sets
 * FP8_DEV_NONFINITE. Requires K % 16 == 0 and 16-byte aligned byte arrays.
 * w8 may alias w8_fnuz and s_ch may alias s_fnuz (in-place conversion).
 */
fp8_status fp8_convert_fnuz(const uint8_t* w8_fnuz, const float* s_fnuz, int64_t N,
                            int64_t K, uint8_t* w8, float* s_ch, void* stream);

/*
 * fp8_quant_act: per-token dynamic activation quantization. Source: model
 * card header paragraph ("activations quantized to FP8 per token at run
 * time"); sizes article, format table (fp8 = FP8 activations per token).
 *   x    [M, ldx] bf16 (uint16 bit patterns), row pitch ldx >= K elements.
 *   x8   [M, K] uint8 out: E4M3 codes (dense, pitch K).
 *   s_tok [M] float32 out: per-token scales amax/448.
 * Requires K % 16 == 0, ldx % 8 == 0, x and x8 16-byte aligned.
 * Device status: FP8_DEV_NONFINITE when a token row holds NaN/Inf.
 */
fp8_status fp8_quant_act(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, uint8_t* x8,
                         float* s_tok, void* stream);

/*
 * fp8_rowwise_linear: y = (x8 . w8^T) * s_tok * s_ch in bf16. Source: E2B
 * article step 3 and model card ("vLLM picked
 * RowWiseTorchFP8ScaledMMLinearKernel"), row-wise scaled FP8 GEMM.
 *   x8 [M, K] uint8 E4M3, s_tok [M] float32 (per token).
 *   w8 [N, K] uint8 E4M3, s_ch  [N] float32 (per output channel).
 *   y  [M, N] bf16 out (uint16 bit patterns), pitch N.
 * y[m, n] = bf16_rn(fp32(acc[m, n] * s_tok[m]) * s_ch[n]) where acc is the
 * fp32 tensor-core sum over k of dec(x8[m,k]) * dec(w8[n,k]). The sum order
 * is fixed per shape, so results are bit-reproducible run to run.
 * Requires K % 16 == 0 and K <= 65536; x8, w8, y 16-byte aligned.
 * Runs on tcgen05 tensor cores with TMA-staged tiles and a TMEM accumulator;
 * M <= 128 selects a swap-AB variant bound by the weight stream (K split over
 * a thread-block cluster when there are few 128-channel tiles).
 *
 * Launch order (programmatic dependent launch): the GEMM is launched as a
 * programmatic dependent of the preceding grid on the stream. Before it waits
 * for that grid it reads only w8 and s_ch, so these must not be written by a
 * preceding grid that lets dependents launch early
 * (griddepcontrol.launch_dependents) before it has finished writing them; no
 * kernel of this library that writes weights does. The decode variant and the
 * quantizers let the next grid launch early; a grid launched after them with
 * the programmatic attribute must wait (griddepcontrol.wait) before it reads
 * y, x8 or s_tok. Grids launched without the attribute are ordered as usual.
 */
fp8_status fp8_rowwise_linear(const uint8_t* x8, const float* s_tok, const uint8_t* w8,
                              const float* s_ch, int64_t M, int64_t N, int64_t K,
                              uint16_t* y, void* stream);

/*
 * fp8_linear_workspace_bytes: size of the workspace fp8_rowwise_linear_ws
 * can use on the current device (0 where the split below is not available).
 * Per pair of SMs of the persistent GEMM grid one 256 x 256 fp32 tile and
 * 16 flags.
 */
size_t fp8_linear_workspace_bytes(void);

/*
 * fp8_rowwise_linear_ws: fp8_rowwise_linear with a workspace ws of ws_bytes
 * bytes (device memory, 16-byte aligned, zero-filled before its first use;
 * every completed call leaves its flags zero again). When the prefill GEMM's
 * tiles make fewer than eight waves over the SM pairs and the last wave is
 * partial, ws_bytes >= fp8_linear_workspace_bytes() lets the last full wave
 * and the partial one be shared out by k-blocks over all pairs (a stream-K
 * split): a tile cut between two pairs has the accumulator of its later
 * k-blocks written to ws by one pair and added, in k order, by the pair that
 * computed its first k-blocks, which then stores the tile (its waits on the
 * other pair are bounded, FP8_DEV_TIMEOUT after about a second). y has the
 * same contract and bound as fp8_rowwise_linear; the sum order of a split
 * tile differs from the unsplit one, but is fixed per shape and device, so
 * results stay bit-reproducible. With ws NULL, too small, or a shape that
 * does not split, it is fp8_rowwise_linear. Calls that may run at the same
 * time (other streams) need workspaces of their own, and a call that ended
 * with FP8_DEV_TIMEOUT may leave flags set: zero the workspace again before
 * reusing it. Errors: those of fp8_rowwise_linear, and FP8_ERR_ALIGNMENT for a
 * ws that is not 16-byte aligned. No counterpart on the pages: a scheduling
 * choice of this library's GEMM.
 */
fp8_status fp8_rowwise_linear_ws(const uint8_t* x8, const float* s_tok, const uint8_t* w8,
                                 const float* s_ch, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                 void* ws, size_t ws_bytes, void* stream);

/*
 * fp8_linear_bf16: the whole W8A8 linear from bf16 activations: per-token
 * quantization of x (exactly fp8_quant_act) followed by the row-wise GEMM
 * (exactly fp8_rowwise_linear), bit-identical to calling the two. Both are
 * launched as programmatic dependents (see fp8_rowwise_linear): the GEMM's
 * prologue and weight stream start while the quantizer runs, and in a chain
 * of decode linears the next quantizer and GEMM start while this GEMM ends.
 *   x [M, K] bf16 (pitch K); x8 [M, K] uint8 and s_tok [M] float32 are
 *   caller-provided scratch that also receive the quantized activations;
 *   w8, s_ch, y as in fp8_rowwise_linear.
 */
fp8_status fp8_linear_bf16(const uint16_t* x, const uint8_t* w8, const float* s_ch, int64_t M,
                           int64_t N, int64_t K, uint8_t* x8, float* s_tok, uint16_t* y,
                           void* stream);

/*
 * fp8_linear_bf16_siblings: several linears that read the same activations
 * (q, k and v of an attention block; gate and up of an MLP), with x
 * quantized once. Source: E2B article, section "第二步：测这张卡的矩阵乘法"
 * (the whole per-token GEMM set of the model, timed inside one graph).
 *   x [M, K] bf16 (pitch K), quantized once into the caller's x8 [M, K] and
 *   s_tok [M] (as fp8_quant_act); then for i < count: y[i] [M, N[i]] =
 *   fp8_rowwise_linear(x8, s_tok, w8[i], s_ch[i]), each GEMM launched as a
 *   programmatic dependent of the one before, so its prologue and weight
 *   stream start while the previous one ends. Bit-identical to
 *   fp8_linear_bf16 called once per weight.
 *   w8, s_ch, N, y: HOST arrays of `count` (1..16) device pointers / sizes.
 * Requirements per linear as fp8_rowwise_linear.
 */
fp8_status fp8_linear_bf16_siblings(const uint16_t* x, int64_t M, int64_t K, int32_t count,
                                    const uint8_t* const* w8, const float* const* s_ch,
                                    const int64_t* N, uint8_t* x8, float* s_tok,
                                    uint16_t* const* y, void* stream);

/*
 * fp8_cast_e4m3: element-wise fp32 -> E4M3 with the library's encoder
 * (round to nearest even, saturating to +-448, NaN -> 0x7F, zero -> 0x00).
 * The encoding step the quantizers use, exposed for exhaustive testing.
 *   x [n] float32, out [n] uint8. Requires 16-byte aligned x and out.
 */
fp8_status fp8_cast_e4m3(const float* x, int64_t n, uint8_t* out, void* stream);

/* ------------------------------------------------------------------------
 * Mixture-of-experts layer. Source: dev.to "Gemma 4 From E2B to 31B on an AMD
 * MI300X", section "Step 1 - Build the Larger Repacks" (128 experts per layer,
 * fused expert banks split into one gate/up/down FP8 linear per expert, bf16
 * router) and section "Why the Mixture-of-Experts Model Sits Lower" (the
 * fp8_w8a8 fused-MoE expert GEMM, E=128, N=704). Routing decisions are inputs;
 * the library groups, gathers, multiplies, activates and combines.
 * ------------------------------------------------------------------------ */

/*
 * fp8_moe_route: group the (token, slot) pairs by expert.
 *   topk_ids [tokens, top_k] int32: expert of each slot, in [0, num_experts).
 *   perm [tokens*top_k] int32 out: flat index token*top_k + slot of each row of
 *     the expert-sorted order; inside one expert rows ascend by flat index.
 *   inv [tokens*top_k] int32 out: inverse of perm.
 *   offsets [num_experts + 1] int32 out: expert e owns rows offsets[e] ..
 *     offsets[e+1] - 1.
 * Deterministic (no atomics decide positions). 1 <= num_experts <= 1024.
 * Ids out of range set FP8_DEV_BAD_INDEX; perm, inv and offsets are then
 * unspecified (every write stays inside them).
 */
fp8_status fp8_moe_route(const int32_t* topk_ids, int64_t tokens, int32_t top_k,
                         int32_t num_experts, int32_t* perm, int32_t* inv, int32_t* offsets,
                         void* stream);

/*
 * fp8_moe_gather: rows of per-token quantized activations in expert order:
 *   x8_rows[i] = x8[perm[i] / top_k], s_rows[i] = s_tok[perm[i] / top_k].
 *   x8 [tokens, K] uint8, s_tok [tokens] fp32 (from fp8_quant_act); rows =
 *   tokens * top_k. Requires K % 16 == 0, 16-byte aligned x8 / x8_rows. A
 *   perm entry outside [0, rows) gives a zero row and scale and sets
 *   FP8_DEV_BAD_INDEX.
 */
fp8_status fp8_moe_gather(const uint8_t* x8, const float* s_tok, const int32_t* perm,
                          int64_t rows, int64_t K, int32_t top_k, uint8_t* x8_rows,
                          float* s_rows, void* stream);

/*
 * fp8_grouped_linear: per-expert row-wise scaled FP8 GEMM. For each expert e,
 * rows offsets[e] .. offsets[e+1]-1 of x8_rows [M_total, K] (scales s_rows)
 * are multiplied by w8[e] (stacked [num_experts * N, K], K-major, scales
 * s_ch [num_experts * N]) into y [M_total, N] bf16, with the same arithmetic
 * and bound as fp8_rowwise_linear. One persistent tcgen05 kernel walks
 * (expert, row tile, column tile) work items derived on the GPU from
 * offsets: 256-row tiles on pairs of SMs (128-row tiles on single SMs where
 * no pair can be scheduled). Requires K % 16 == 0, num_experts <= 1024;
 * offsets must be non-decreasing within [0, M_total]: an expert whose row
 * range is not (a device-side error) is skipped and sets FP8_DEV_BAD_INDEX.
 */
fp8_status fp8_grouped_linear(const uint8_t* x8_rows, const float* s_rows, const int32_t* offsets,
                              int32_t num_experts, int64_t M_total, const uint8_t* w8,
                              const float* s_ch, int64_t N, int64_t K, uint16_t* y, void* stream);

/*
 * fp8_moe_interleave_gate_up: the gate/up weights of fp8_grouped_linear_geglu,
 * a load-time reordering. w8 [num_experts, 2*inter, K] uint8 E4M3 (per
 * expert the gate rows 0..inter-1, then the up rows) and s_ch
 * [num_experts, 2*inter] fp32 become w8_il [num_experts, 256*T, K] and s_il
 * [num_experts, 256*T], T = ceil(inter / 128): row t*256 + s*128 + j of an
 * expert is its gate (s = 0) or up (s = 1) row of feature t*128 + j; features
 * >= inter give zero rows with scale 0. Requires K % 16 == 0, inter % 16 ==
 * 0; 16-byte aligned w8 and w8_il. No counterpart on the pages: a layout for
 * the fused GeGLU below.
 */
fp8_status fp8_moe_interleave_gate_up(const uint8_t* w8, const float* s_ch, int32_t num_experts,
                                      int64_t inter, int64_t K, uint8_t* w8_il, float* s_il,
                                      void* stream);

/*
 * fp8_grouped_linear_geglu: the expert gate/up GEMM with the GeGLU unit in
 * its epilogue. For each expert e and each of its rows i (offsets as in
 * fp8_grouped_linear): gate and up are the row-wise scaled FP8 products of
 * x8_rows[i] with the expert's gate and up rows, each rounded to bf16 exactly
 * as fp8_grouped_linear stores them, and h [M_total, inter] bf16 receives
 * bf16(gelu_tanh(gate) * up) - bit for bit what fp8_moe_geglu_quant writes
 * to h_out from fp8_grouped_linear's output. Quantize h with fp8_quant_act
 * (the same per-row quantization as fp8_moe_geglu_quant). w8_il / s_il in
 * the layout of fp8_moe_interleave_gate_up (s_il 16-byte aligned). Requires
 * inter % 16 == 0, K % 16 == 0; runs on CTA pairs (FP8_ERR_UNSUPPORTED if
 * the device cannot co-schedule them). No counterpart on the pages beyond
 * the expert MLP itself (readings as for fp8_moe_geglu_quant).
 */
fp8_status fp8_grouped_linear_geglu(const uint8_t* x8_rows, const float* s_rows,
                                    const int32_t* offsets, int32_t num_experts, int64_t M_total,
                                    const uint8_t* w8_il, const float* s_il, int64_t inter,
                                    int64_t K, uint16_t* h, void* stream);

/*
 * fp8_moe_geglu_quant: h = bf16(gelu_tanh(gate) * up) per element of
 * gate_up [M, 2*inter] bf16 (gate in columns 0..inter-1, up after it; fp32
 * arithmetic, one rounding to bf16), then per-row E4M3 quantization of h with
 * the contract above: h8 [M, inter] uint8, s_h [M] fp32. h_out [M, inter]
 * bf16 receives h when not NULL. Requires inter % 16 == 0.
 */
fp8_status fp8_moe_geglu_quant(const uint16_t* gate_up, int64_t M, int64_t inter, uint8_t* h8,
                               float* s_h, uint16_t* h_out, void* stream);

/*
 * fp8_moe_combine: out[t] = sum_{j<top_k} w[t,j] * rows[inv[t*top_k + j]]
 * (fp32 products and sums in slot order, one rounding to bf16); rows
 * [tokens*top_k, H] bf16 in expert order, weights [tokens, top_k] fp32 or
 * NULL for 1/top_k. Requires H % 8 == 0 and 1 <= top_k <= 16. An inv entry
 * outside [0, tokens*top_k) contributes nothing and sets FP8_DEV_BAD_INDEX.
 */
fp8_status fp8_moe_combine(const uint16_t* rows, const int32_t* inv, int64_t tokens,
                           int32_t top_k, int64_t H, const float* weights, uint16_t* out,
                           void* stream);

/*
 * bf16_linear: y = x . w^T with bf16 operands, fp32 tensor-core accumulation
 * (kind::f16) and one rounding to bf16; no scales. The router of the
 * mixture-of-experts layer, router.proj, stays bf16 in every build (sizes
 * article, "Step 1 - Build the Larger Repacks"); the W4A16 build's long-M
 * path multiplies by its weights unpacked to bf16 (w4a16_linear).
 *   x [M, K] bf16, w [N, K] bf16, y [M, N] bf16 out; pitch K and N.
 * The same kernels and launch order as fp8_rowwise_linear. Requires K % 8
 * == 0 and K <= 32768; x, w, y 16-byte aligned.
 */
fp8_status bf16_linear(const uint16_t* x, const uint16_t* w, int64_t M, int64_t N, int64_t K,
                       uint16_t* y, void* stream);

/*
 * fp8_moe_topk: the router's expert choice from its bf16 logits.
 *   logits [tokens, num_experts] bf16; ids [tokens, top_k] int32 out: the
 *   top_k largest logits' experts in descending order of logit, ties to the
 *   lower expert index (unique); weights [tokens, top_k] fp32 out: the
 *   softmax over the chosen logits, exp(l_j - l_max) / sum_i exp(l_i - l_max)
 *   (fp32, sum in slot order, IEEE division). The pages give no router
 *   weights; the renormalized top-k softmax is the reading used.
 * Requires 1 <= top_k <= 16, top_k <= num_experts <= 1024. A NaN or infinite
 * logit sets FP8_DEV_NONFINITE; that token's outputs are unspecified.
 */
fp8_status fp8_moe_topk(const uint16_t* logits, int64_t tokens, int32_t num_experts, int32_t top_k,
                        int32_t* ids, float* weights, void* stream);

/* ------------------------------------------------------------------------
 * W4A16 build. Source: dev.to "Gemma 4 From E2B to 31B on an AMD MI300X",
 * section "The Sizes and the Builds" (q4w4a16: int4 holding the QAT grid
 * exactly, bf16 activations) and section "The 4-Bit Builds Stay Slow at
 * Every Size" (the weights are unpacked to bf16 before each multiply); E2B
 * article, section "十种构建" (the 4-bit repack stores the QAT values as int4
 * with each group's trained step, without rounding again).
 *
 * The weights are the QAT q4_0 tensors themselves: q4 [N, K/2] packed int4
 * and d [N, K/32] fp32, as fp8_repack_qat takes them. They are unpacked to
 * w = bf16_rn(fp32(d * q)) and multiplied with bf16 tensor-core MMAs
 * (fp32 accumulation): |y - y_exact| <= 4e-3 sum_k |x w| + 1 bf16 ulp,
 * y_exact = sum_k x d q.
 * ------------------------------------------------------------------------ */

/*
 * w4a16_dequant: w [N, K] bf16 out = bf16_rn(fp32(d[n, k/32] * q[n, k])),
 * bit-exact. Requires K % 32 == 0, K <= 32768; q4 and w 16-byte aligned.
 */
fp8_status w4a16_dequant(const uint8_t* q4, const float* d, int64_t N, int64_t K, uint16_t* w,
                         void* stream);

/*
 * w4a16_workspace_bytes: the workspace w4a16_linear needs for this shape:
 * 0 when M <= 128 and K % 128 == 0 (the weights are unpacked on chip, inside
 * the GEMM), else N * K * 2 bytes (the unpacked bf16 weights).
 */
size_t w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * w4a16_linear: y = x . w^T, x [M, K] bf16 (pitch K), y [M, N] bf16 out.
 * M <= 128 with K % 128 == 0: one kernel streams q4 and d (0.625 bytes per
 * weight) and unpacks them in shared memory for the MMA (swap-AB, K split
 * over a cluster for narrow layers). Otherwise w4a16_dequant into w_ws
 * (ws_bytes >= w4a16_workspace_bytes; caller-owned) followed by
 * bf16_linear. Requires K % 32 == 0, K <= 32768; x, y, w_ws 16-byte aligned.
 * FP8_ERR_INVALID_ARG when a needed workspace is missing or too small.
 */
fp8_status w4a16_linear(const uint16_t* x, const uint8_t* q4, const float* d, int64_t M, int64_t N,
                        int64_t K, uint16_t* y, uint16_t* w_ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * int8 W8A8 build. Source: dev.to "Gemma 4 From E2B to 31B on an AMD MI300X",
 * section "The Sizes and the Builds" (format table: w8a8 = int8 weights per
 * channel, int8 activations per token, from the same QAT release); E2B
 * article, section "它们离训练权重有多近？" (the int8 build rounds every value
 * to one of 255 levels per row) and section "第二步：测这张卡的矩阵乘法" (the
 * int8 GEMM at M = 64; PyTorch's int8 matmul there refuses M < 17 - these
 * calls accept every M >= 1).
 *
 * Quantization contract (bit-exact): per row, amax = max |v|,
 * s = fp32(amax / 127) (IEEE division), code = clamp(RNE(fp32(v / s)), -127,
 * 127) as int8 (round half to even); an all-zero row gets s = 0 and zero
 * codes. GEMM contract (bit-exact): acc = the exact int32 sum of the int8
 * products (tensor-core kind::i8), y = bf16_rn(fp32(fp32(fp32(acc) * s_tok)
 * * s_ch)) with one IEEE rounding per step.
 * ------------------------------------------------------------------------ */

/*
 * int8_repack_qat: QAT q4_0-grid weights -> per-output-channel int8.
 *   q4 [N, K/2] uint8 and d [N, K/32] float32 as in fp8_repack_qat (values
 *   w = fp32(d * q)); w8 [N, K] int8 out; s_ch [N] float32 out.
 * Requires K % 32 == 0; q4, d, w8 16-byte aligned. Device status:
 * FP8_DEV_NONFINITE when a row's d*q is not finite.
 */
fp8_status int8_repack_qat(const uint8_t* q4, const float* d, int64_t N, int64_t K, int8_t* w8,
                           float* s_ch, void* stream);

/*
 * int8_quant_act: per-token int8 quantization of bf16 activations.
 *   x [M, ldx] bf16 (pitch ldx >= K), x8 [M, K] int8 out, s_tok [M] fp32 out.
 * Requires K % 16 == 0, ldx % 8 == 0, x and x8 16-byte aligned. Device
 * status: FP8_DEV_NONFINITE when a token row holds NaN/Inf.
 */
fp8_status int8_quant_act(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int8_t* x8,
                          float* s_tok, void* stream);

/*
 * int8_rowwise_linear: y = (x8 . w8^T) * s_tok * s_ch in bf16 (contract
 * above). x8 [M, K] int8, s_tok [M], w8 [N, K] int8, s_ch [N], y [M, N] bf16.
 * The same kernels, tiles and launch order as fp8_rowwise_linear (see its
 * notes on programmatic dependent launch), with int8 operands and int32
 * accumulators. Requires K % 16 == 0, K <= 65536; x8, w8, y 16-byte aligned.
 */
fp8_status int8_rowwise_linear(const int8_t* x8, const float* s_tok, const int8_t* w8,
                               const float* s_ch, int64_t M, int64_t N, int64_t K, uint16_t* y,
                               void* stream);

/*
 * int8_rowwise_linear_ws: int8_rowwise_linear with the workspace and the
 * k-block split of fp8_rowwise_linear_ws (same workspace contract). The
 * parts are int32 sums, added exactly, so y is bit for bit that of
 * int8_rowwise_linear.
 */
fp8_status int8_rowwise_linear_ws(const int8_t* x8, const float* s_tok, const int8_t* w8,
                                  const float* s_ch, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                  void* ws, size_t ws_bytes, void* stream);

/*
 * int8_linear_bf16: int8_quant_act of x (pitch K) into the caller's x8 /
 * s_tok, then int8_rowwise_linear; bit-identical to the two calls.
 */
fp8_status int8_linear_bf16(const uint16_t* x, const int8_t* w8, const float* s_ch, int64_t M,
                            int64_t N, int64_t K, int8_t* x8, float* s_tok, uint16_t* y,
                            void* stream);

/*
 * fp8_linear_bf16_noalloc: the same computation as fp8_linear_bf16 (per-token
 * quantization of x, then the row-wise FP8 GEMM, with bit-identical results),
 * for callers that cannot provide the quantized-activation scratch buffers.
 * The pages have no counterpart to this entry point; it exists for callers
 * that must not allocate device memory at all, for example a plugin that a
 * host framework hands nothing but fixed input and output buffers because
 * that framework owns all of device memory, or a latency-critical serving
 * loop that cannot afford cudaMalloc's implicit device-wide synchronization.
 *
 *   x [M, K] bf16 (pitch K), w8 [N, K] E4M3, s_ch [N] fp32, y [M, N] bf16 out:
 *   as in fp8_linear_bf16.
 *
 * Scratch: the quantized activations (M*K bytes, rounded up to 256) and the
 * per-token scales (4*M bytes) live in one file-scope device array of
 * FP8_NOALLOC_SCRATCH_BYTES bytes that every GPU which loads this library
 * holds until the process exits. Larger problems return
 * FP8_ERR_SCRATCH_LIMIT before anything is enqueued. The call allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *
 * All calls share that one array and it keeps the last call's contents
 * (nothing in it needs to start at zero: each call writes the scratch it
 * reads). Calls that can overlap on the GPU - on different streams, or on
 * different host threads without ordering - race on the array and must be
 * serialized by the caller.
 *
 * The first call on each device looks up that device's address of the array
 * (cudaGetSymbolAddress, with that device current) and caches it for the
 * life of the process (see the conventions above: no cudaDeviceReset); make
 * that first call before any stream capture begins.
 */
#define FP8_NOALLOC_SCRATCH_BYTES (4u << 20)
fp8_status fp8_linear_bf16_noalloc(const uint16_t* x, const uint8_t* w8, const float* s_ch,
                                   int64_t M, int64_t N, int64_t K, uint16_t* y, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8W8A8_H */
