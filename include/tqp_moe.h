/*
 * tqp_moe.h - C ABI of the B200 (sm_100a) TQP MoE layer and its reversible coupling.
 *
 * The layer is the routed-expert block of the reversible sparse MoE described in
 * "Reversible Sparse MoE Single Node" (skills-directory page) and the abstract
 * of "Reversible Foundations: Training a 120B Sparse MoE through
 * State-Preserving Scaling":
 *   - 460 routed experts with top-12 routing ("Architecture Details"; Abstract),
 *   - TQP: frozen quantised base expert weights plus trained low-rank adapters
 *     per expert, full-precision router ("Principle 3: TQP Optimizer Strategy";
 *     "TQP Quantization"; Abstract, "Single-node economics"),
 *   - stateless routing, recomputed during the inverse ("Reversibility
 *     Implementation"),
 *   - reversible residual blocks whose inverse is a subtraction, used to
 *     reconstruct activations in the backward pass instead of storing them
 *     ("Principle 1: Reversible Recurrence Stack"; "Pattern 1"; Abstract,
 *     "Reversibility").
 * The pages fix neither equations nor formats; the readings used here are:
 * gates = softmax over the k chosen fp32 logits (ties -> lower expert id),
 * SwiGLU experts, LoRA W' = W + s*A*B on gate, up and down, symmetric int4
 * base weights with one bf16 scale per group of `group` input positions, and
 * the additive coupling y1 = x1 + F(x2), y2 = x2 + G(y1).
 *
 * Conventions (all entry points)
 *   - Return value: TQP_OK (0) or a negative TQP_ERR_* code. Argument errors
 *     are detected on the host before anything is enqueued.
 *   - Data-dependent errors are OR-ed asynchronously into `dev_status`, a
 *     caller-owned int32 in device memory that the caller zeroes and reads
 *     after synchronising (nullable: then they are not reported):
 *       TQP_STATUS_NONFINITE  a NaN/Inf router logit or input; an x value
 *                             outside the fp16 range; an fp16 intermediate of
 *                             the expert path (H, the kept G|U, O, s X A,
 *                             s H A, and in the backward dO, dG|dU, dX and the
 *                             rank-space products) that overflowed; a LoRA
 *                             factor outside the fp16 range. Outputs are then
 *                             unreliable.
 *       TQP_STATUS_BAD_ID     an expert id outside [0, E), or one token listing
 *                             the same expert twice.
 *       TQP_STATUS_TIMEOUT    a device-side wait hit its limit; outputs are then
 *                             undefined.
 *       TQP_STATUS_RANGE      a nonzero group scale outside [2^-17, 8192): the
 *                             products q * scale are then not all exact in fp16
 *                             (the expert contractions run on exact fp16 weights
 *                             otherwise); or, in the coupling and stack calls, a
 *                             stream value of magnitude 256 or more (or not
 *                             finite): the stream adds are then no longer exact.
 *     Nothing traps, prints or exits.
 *   - Every pointer argument is caller-owned DEVICE memory (unless stated),
 *     16-byte aligned, dense row-major. The library never allocates device
 *     memory: scratch comes from `ws` of at least the size returned by the
 *     matching *_workspace_size query (which needs no GPU).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns at once. Calls hold no global state and may
 *     run concurrently on different streams with disjoint workspaces (the two
 *     exceptions are named where they are declared: moe_permute_noalloc's fixed
 *     scratch and the tqp_debug_set_wait_limit_ns test hook).
 *   - bf16 tensors are uint16_t bit patterns.
 *   - Outputs are overwritten (never accumulated into).
 *
 * Weight formats (one tqp_moe_weights per layer; p = 0 gate, 1 up, 2 down;
 * in_p / out_p = d / ffn for gate and up, ffn / d for down)
 *   router_w   [E][d] fp32.
 *   router_bias[E] fp32 or NULL: additive per-expert bias, added to the logits
 *              before top-k and gates.
 *   wq[p]      bits = 4: [E][out_p][in_p/2] uint8: int4 codes of the frozen base
 *              weight W_p[out][in]. Each little-endian 32-bit word holds 8
 *              consecutive input positions k0..k7 of one output row as
 *              two's-complement nibbles: k(2i) in bits [4i,4i+4), k(2i+1) in bits
 *              [16+4i,16+4i+4).
 *              bits = 8: [E][out_p][in_p] int8 codes (two's complement), one per
 *              input position (TQP Quantization: base weights int8 or int4).
 *   wscale[p]  [E][in_p/group][out_p] bf16: W_p[n][k] = q[n][k] * wscale[k/group][n].
 *   lora_a[p]  [E][rank][in_p] bf16: A_p^T.
 *   lora_b[p]  [E][out_p][rank] bf16: B_p^T.
 *   The projection is  x -> x W_p^T + lora_scale * (x A_p) B_p.
 *
 * Exactness: int4 codes times bf16 scales are exact in fp16, so the expert
 * contractions run on the exact dequantised weights; int8 codes times bf16
 * scales (up to 15 significant bits) are rounded once to fp16 (relative error
 * at most 2^-11 per weight).
 *
 * Validity (host-checked, else TQP_ERR_INVALID_ARG / TQP_ERR_UNSUPPORTED):
 *   bits in {0, 4, 8}, and ffn % 128 == 0 for bits = 8;
 *   1 <= top_k <= E <= 4096; d % 128 == 0; ffn % 64 == 0; 64 <= d, ffn <= 16384;
 *   group in {32, 64, 128, 256} dividing d and ffn; rank % 8 == 0 and
 *   0 <= rank <= 64 (rank 0 skips the adapter path); T >= 0 (T == 0 is a no-op).
 */
#ifndef TQP_MOE_H_
#define TQP_MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TQP_OK 0
#define TQP_ERR_INVALID_ARG (-1)
#define TQP_ERR_UNSUPPORTED (-2)
#define TQP_ERR_WORKSPACE (-3)
#define TQP_ERR_CUDA (-4)

#define TQP_STATUS_NONFINITE 1
#define TQP_STATUS_BAD_ID 2
#define TQP_STATUS_TIMEOUT 4
#define TQP_STATUS_RANGE 8

#define TQP_DTYPE_BF16 0
#define TQP_DTYPE_F32 1

typedef struct tqp_moe_weights {
  int E;            /* routed experts */
  int d;            /* model width */
  int ffn;          /* expert SwiGLU hidden width */
  int group;        /* quantisation group along the input dimension */
  int rank;         /* LoRA rank */
  int top_k;        /* experts per token */
  float lora_scale; /* s = alpha / rank */
  const float* router_w;
  const float* router_bias;
  const uint8_t* wq[3];
  const uint16_t* wscale[3];
  const uint16_t* lora_a[3];
  const uint16_t* lora_b[3];
  int bits;         /* base-weight code width: 4 (0 also means 4) or 8 */
} tqp_moe_weights;

/* Adapter gradients of one layer, fp32, same layouts as lora_a / lora_b:
 * dA[p] [E][rank][in_p], dB[p] [E][out_p][rank]. Overwritten. */
typedef struct tqp_adapter_grads {
  float* dA[3];
  float* dB[3];
} tqp_adapter_grads;

/* Library version (major*10000 + minor*100 + patch) and error names. */
int tqp_version(void);
const char* tqp_error_string(int code);

/* ---------------------------------------------------------------------------
 * moe_router_gemm: router logits at full precision (the TQP Quantization list
 * keeps the router unquantised because routing quality depends on it).
 *   logits[t][e] = sum_i x[t][i] * router_w[e][i] (+ router_bias[e]), accurate to
 *   fp32 (the fp32 weights are split exactly into three bf16 parts and the
 *   products accumulated in fp32 on the tensor cores).
 *   x [T][d] bf16; logits [T][E] fp32. ws: moe_router_gemm_workspace_size.
 * ------------------------------------------------------------------------- */
size_t moe_router_gemm_workspace_size(int T, const tqp_moe_weights* w);
int moe_router_gemm(const uint16_t* x, int T, const tqp_moe_weights* w, float* logits, void* ws,
                    size_t ws_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * moe_route: top-k expert selection and gates ("Top-12 routing", Architecture
 * Details; stateless, so a replay from the same logits gives the same ids).
 *   ids[t][j]: the k experts with the largest logits, in descending order;
 *   exact ties -> lower id first; +0.0 ties with -0.0; NaN ranks lowest.
 *   gates[t][j] = exp(l_j - l_0) / sum_j' exp(l_j' - l_0) over the chosen ones.
 *   A NaN or +-Inf logit anywhere in the row raises TQP_STATUS_NONFINITE.
 *   logits [T][E] fp32; ids [T][k] int32; gates [T][k] fp32.
 * ------------------------------------------------------------------------- */
int moe_route(const float* logits, int T, int E, int k, int32_t* ids, float* gates, int32_t* dev_status,
              void* stream);

/* ---------------------------------------------------------------------------
 * moe_permute: stable counting sort of the T*k assignments by expert (the
 * dispatch step of sparse MoE routing, "Related Methods": Switch, GShard).
 *   offsets[e] = #assignments to experts < e, offsets[E] = T*k;
 *   rows of one expert are in increasing token order;
 *   perm_token[row] = token of that row; inv[t*k + j] = row of assignment (t, j).
 *   Precondition: each token's k ids are distinct (moe_route guarantees it).
 *   ids outside [0, E), and a token that lists one expert twice, raise
 *   TQP_STATUS_BAD_ID; the outputs are then not a valid permutation.
 *   ws: moe_permute_workspace_size.
 * ------------------------------------------------------------------------- */
size_t moe_permute_workspace_size(int T, int E, int k);
int moe_permute(const int32_t* ids, int T, int E, int k, int32_t* offsets, int32_t* perm_token, int32_t* inv,
                void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * moe_permute_noalloc: moe_permute for callers that cannot allocate device
 * memory (a runtime that only hands out memory from its own fixed pool, a
 * serving process that must never block in the driver's allocator, code with
 * nowhere to keep a workspace between calls). The pages have no counterpart:
 * this is a library convenience, not part of the method.
 *   Same arguments and results as moe_permute, minus the workspace: the
 *   scratch lives in a fixed array inside this library's device image, of
 *   moe_permute_noalloc_max_bytes() bytes (about 1 MiB), which every GPU that
 *   loads the library holds until the process exits.
 *   Limits: T <= 16384 and E <= 512, else TQP_ERR_UNSUPPORTED (nothing is
 *   enqueued). Allocates nothing: no cudaMalloc, no cudaFree, no allocating
 *   library call.
 *   The first call under each CUDA context looks up the array's device address
 *   in that context with the device current (cudaGetSymbolAddress) and caches
 *   it under the context's unique id, so a context created after a device
 *   reset, or a second context on the device, gets its own lookup; make the
 *   first call in a context before any stream capture.
 *   All calls share the one array, and every call overwrites it before reading
 *   it; calls that overlap on the GPU (concurrent streams) race on it and must
 *   be serialised by the caller.
 * ------------------------------------------------------------------------- */
size_t moe_permute_noalloc_max_bytes(void);
int moe_permute_noalloc(const int32_t* ids, int T, int E, int k, int32_t* offsets, int32_t* perm_token,
                        int32_t* inv, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * tqp_grouped_ffn: the routed experts (Pattern 3: low-rank adapters trained per
 * expert over frozen quantised base expert weights). For each expert e and each
 * of its rows (row r holds token perm_token[r]):
 *   G = X Wg^T + s (X Ag) Bg ;  U = X Wu^T + s (X Au) Bu ;  H = fp16(silu(G) * U)
 *   O = fp16(H Wd^T + s (H Ad) Bd)
 * The int4 base is dequantised exactly to fp16 (q * scale) and every
 * contraction runs on the tensor cores (fp16 x fp16 -> fp32); the adapter
 * products s X A and s H A are kept in fp16.
 *   x [T][d] bf16 (tokens, gathered through perm_token); offsets [E+1];
 *   h [T*k][ffn] fp16 output (permuted row order; kept for the backward);
 *   out_perm [T*k][d] fp16 output (permuted row order).
 *   ws: tqp_grouped_ffn_workspace_size. Errors: as the conventions above (x
 *   values and fp16 intermediates outside the fp16 range raise
 *   TQP_STATUS_NONFINITE, group scales outside the exact range TQP_STATUS_RANGE).
 *
 * tqp_grouped_ffn_part: the same computation issued one part at a time, for a
 * caller that times or overlaps the parts. Parts must be issued in order
 * TQP_FFN_PREPARE, TQP_FFN_GATE_UP, TQP_FFN_RANK, TQP_FFN_DOWN with the same
 * arguments and workspace; together they equal one tqp_grouped_ffn call.
 *   TQP_FFN_PREPARE : expert block schedule, x and Ad in fp16, s X [Ag|Au]
 *   TQP_FFN_GATE_UP : h (one kernel: the gate/up expert contraction + SwiGLU)
 *   TQP_FFN_RANK    : s H Ad
 *   TQP_FFN_DOWN    : out_perm (one kernel: the down expert contraction)
 * Returns TQP_ERR_INVALID_ARG for an unknown part.
 * ------------------------------------------------------------------------- */
#define TQP_FFN_PREPARE 0
#define TQP_FFN_GATE_UP 1
#define TQP_FFN_RANK 2
#define TQP_FFN_DOWN 3
size_t tqp_grouped_ffn_workspace_size(int T, const tqp_moe_weights* w);
int tqp_grouped_ffn(const uint16_t* x, int T, const int32_t* offsets, const int32_t* perm_token,
                    const tqp_moe_weights* w, uint16_t* h, uint16_t* out_perm, void* ws, size_t ws_bytes,
                    int32_t* dev_status, void* stream);
int tqp_grouped_ffn_part(int part, const uint16_t* x, int T, const int32_t* offsets, const int32_t* perm_token,
                         const tqp_moe_weights* w, uint16_t* h, uint16_t* out_perm, void* ws, size_t ws_bytes,
                         int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * moe_combine: gate-weighted un-permute (scatter back to tokens), plus the
 * additive coupling when a residual is given ("Pattern 1": addition and
 * subtraction are the invertible primitives).
 *   m[t] = bf16( sum_{j<k} gates[t][j] * out_perm[inv[t*k + j]] )  (out_perm fp16 as
 *   written by tqp_grouped_ffn; fixed j order, fp32 accumulation, no atomics:
 *   deterministic)
 *   y[t] = m[t]                         if residual == NULL
 *   y[t] = residual[t] + sign * m[t]    otherwise (fp32 arithmetic)
 *   residual_dtype / y_dtype: TQP_DTYPE_BF16 or TQP_DTYPE_F32 (bf16 output is
 *   rounded to nearest even). y_bf16 (nullable): extra bf16 copy of y.
 * ------------------------------------------------------------------------- */
int moe_combine(const uint16_t* out_perm, const int32_t* inv, const float* gates, int T, int k, int d,
                const void* residual, int residual_dtype, float sign, void* y, int y_dtype, uint16_t* y_bf16,
                void* stream);

/* ---------------------------------------------------------------------------
 * tqp_moe_layer_fwd: router GEMM -> route -> permute -> grouped FFN -> combine.
 *   x [T][d] bf16 -> y [T][d] bf16 (the MoE output, no residual).
 *   ws: tqp_moe_layer_workspace_size.
 * ------------------------------------------------------------------------- */
size_t tqp_moe_layer_workspace_size(int T, const tqp_moe_weights* w);
int tqp_moe_layer_fwd(const uint16_t* x, int T, const tqp_moe_weights* w, uint16_t* y, void* ws,
                      size_t ws_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * Reversible additive coupling ("Principle 1"; "Reversibility
 * Implementation": reversible residual blocks, RevNet).
 *   rev_couple_fwd: y1 = x1 + F(x2); y2 = x2 + G(bf16(y1)).
 *     x1, x2 [T][d] bf16 in; y1, y2 [T][d] fp32 out.
 *   rev_couple_inv: x2 = y2 - G(bf16(y1)); x1 = y1 - F(x2), rounded to bf16.
 *     y1, y2 fp32 in; x1, x2 bf16 out. Routing is recomputed (stateless).
 *   Stream format: the streams are fp32 multiples of 2^-16 below 256 in
 *   magnitude ("the grid"). x1, x2 and each layer's bf16 branch output are
 *   rounded to the grid (half to even) before the add; F reads x2 on the
 *   grid. On the grid every add and subtract is exact in fp32, and the layers
 *   are deterministic, so rev_couple_inv returns x1, x2 on the grid bit for
 *   bit: x itself wherever |x| >= 2^-9, else x moved by at most 2^-17. The
 *   inverse rounds its inputs y1, y2 to the grid as well (a no-op on the
 *   outputs of rev_couple_fwd). A stream value leaving the range raises
 *   TQP_STATUS_RANGE.
 *   F and G must share d. ws: rev_couple_workspace_size (both calls).
 * ------------------------------------------------------------------------- */
size_t rev_couple_workspace_size(int T, const tqp_moe_weights* F, const tqp_moe_weights* G);
int rev_couple_fwd(const uint16_t* x1, const uint16_t* x2, int T, const tqp_moe_weights* F,
                   const tqp_moe_weights* G, float* y1, float* y2, void* ws, size_t ws_bytes,
                   int32_t* dev_status, void* stream);
int rev_couple_inv(const float* y1, const float* y2, int T, const tqp_moe_weights* F, const tqp_moe_weights* G,
                   uint16_t* x1, uint16_t* x2, void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * tqp_moe_layer_bwd: gradients of <dy, layer(x)>. The base weights stay fixed
 * in their quantised form and the router is frozen, so only the adapters get
 * gradients (TQP Quantization; Principle 3 keeps optimizer state on the
 * adapters alone).
 *   x [T][d] bf16; dy [T][d] fp32 -> dx [T][d] fp32 (through the experts and,
 *   via the softmax over the chosen logits, through the frozen router), and the
 *   adapter gradients `grads`. Top-k selection is treated as constant.
 *   grads: dA[p] [E][r][in_p], dB[p] [E][out_p][r] fp32, caller-owned device
 *   memory, overwritten (not accumulated). With rank > 0 each must be non-null
 *   and 16-byte aligned, else TQP_ERR_INVALID_ARG before any launch; ffn must be
 *   a multiple of 128, else TQP_ERR_UNSUPPORTED.
 *   The fp16 intermediates are computed for dy * 2^P, with the power of two P
 *   chosen from max|dy| on the device so that dO = gate * dy * 2^P peaks near
 *   2^8; the gradients are scaled back by 2^-P in fp32. The result therefore
 *   does not depend on the magnitude of dy (no fp16 underflow or overflow for
 *   small or large cotangents).
 *   ws: tqp_moe_layer_bwd_workspace_size (the layer's forward workspace plus
 *   G|U, dG|dU, dO, dha, dxa, the rank-space B operand and a row copy of the
 *   adapter A factors in fp16).
 * ------------------------------------------------------------------------- */
size_t tqp_moe_layer_bwd_workspace_size(int T, const tqp_moe_weights* w);
int tqp_moe_layer_bwd(const uint16_t* x, const float* dy, int T, const tqp_moe_weights* w, float* dx,
                      const tqp_adapter_grads* grads, void* ws, size_t ws_bytes, int32_t* dev_status,
                      void* stream);

/* ---------------------------------------------------------------------------
 * tqp_adapter_bwd: reversible block backward from the block outputs only
 * (Principle 1: the backward pass rebuilds each block's inputs from its
 * outputs and takes that block's gradients locally).
 *   G-step: z = bf16(y1); x2 = y2 - G(z); G's adapter grads for cotangent dy2;
 *           dz1 = dy1 + J_G(z)^T dy2.
 *   F-step: x1 = y1 - F(x2); F's adapter grads for cotangent dz1;
 *           dx2 = dy2 + J_F(x2)^T dz1; dx1 = dz1.
 *   y1, y2, dy1, dy2 [T][d] fp32 in; x1, x2 [T][d] bf16 out (reconstructed);
 *   dx1, dx2 [T][d] fp32 out; gF, gG adapter gradients of F and G (both
 *   checked on the host, as for tqp_moe_layer_bwd, before any launch).
 *   Each layer's backward reuses the routing and intermediates of the inverse
 *   step that ran that layer's forward, so no layer forward runs twice.
 *   ws: tqp_adapter_bwd_workspace_size.
 * ------------------------------------------------------------------------- */
size_t tqp_adapter_bwd_workspace_size(int T, const tqp_moe_weights* F, const tqp_moe_weights* G);
int tqp_adapter_bwd(const float* y1, const float* y2, const float* dy1, const float* dy2, int T,
                    const tqp_moe_weights* F, const tqp_moe_weights* G, uint16_t* x1, uint16_t* x2, float* dx1,
                    float* dx2, const tqp_adapter_grads* gF, const tqp_adapter_grads* gG, void* ws,
                    size_t ws_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * Reversible stack of L coupling blocks (Principle 1: Reversible Recurrence
 * Stack; Key Innovation: activation memory stays flat as the model deepens).
 * Block l maps streams (a1, a2) to
 *   b1 = a1 + F_l(bf16(a2)),   b2 = a2 + G_l(bf16(b1)).
 * Block 0's inputs are x1, x2 (bf16); the streams between blocks are carried
 * in fp32 on the coupling's grid (each layer reads the bf16 rounding of its
 * stream), so the inverse is exact at any depth; the outputs of block L-1 are
 * y1, y2 (fp32). With L = 1 this is rev_couple_fwd exactly.
 *   F, G: arrays of L weight sets (all with the same d).
 *   rev_stack_fwd: x1, x2 [T][d] bf16 -> y1, y2 [T][d] fp32.
 *   rev_stack_inv: y1, y2 -> x1, x2 (bf16), walking the blocks from L-1 down
 *     with a2 = b2 - G_l(bf16(b1)), a1 = b1 - F_l(bf16(a2)); routing is
 *     recomputed (stateless).
 *   rev_stack_bwd: the backward of the whole stack from its outputs alone: for
 *     l = L-1 .. 0 it reconstructs block l's inputs from its outputs and takes
 *     that block's gradients (each layer's backward reuses the routing and
 *     intermediates of the inverse step that just ran its forward), so no
 *     block's activations are stored. In: y1, y2, dy1, dy2 [T][d] fp32. Out:
 *     x1, x2 (bf16, reconstructed inputs of block 0), dx1, dx2 [T][d] fp32, and
 *     the adapter gradients of every layer: gF[l], gG[l] (arrays of L structs,
 *     each checked as for tqp_moe_layer_bwd; overwritten). Every ffn must be a
 *     multiple of 128 (else TQP_ERR_UNSUPPORTED).
 *   ws: rev_stack_workspace_size (the same size serves all three calls). It
 *   holds two sets of four fp32 stream buffers, two bf16 layer inputs, one
 *   fp32 input gradient and one layer's forward + backward workspace: it does
 *   not grow with L. 1 <= L <= 4096.
 * ------------------------------------------------------------------------- */
size_t rev_stack_workspace_size(int T, int L, const tqp_moe_weights* const* F, const tqp_moe_weights* const* G);
int rev_stack_fwd(const uint16_t* x1, const uint16_t* x2, int T, int L, const tqp_moe_weights* const* F,
                  const tqp_moe_weights* const* G, float* y1, float* y2, void* ws, size_t ws_bytes,
                  int32_t* dev_status, void* stream);
int rev_stack_inv(const float* y1, const float* y2, int T, int L, const tqp_moe_weights* const* F,
                  const tqp_moe_weights* const* G, uint16_t* x1, uint16_t* x2, void* ws, size_t ws_bytes,
                  int32_t* dev_status, void* stream);
int rev_stack_bwd(const float* y1, const float* y2, const float* dy1, const float* dy2, int T, int L,
                  const tqp_moe_weights* const* F, const tqp_moe_weights* const* G, uint16_t* x1, uint16_t* x2,
                  float* dx1, float* dx2, const tqp_adapter_grads* const* gF, const tqp_adapter_grads* const* gG,
                  void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * tqp_adamw_step: one optimizer step over adapter parameters (Principle 3 and
 * Pattern 3: optimizer state lives on the adapters only; the pages do not name
 * the optimizer, this is AdamW with decoupled weight decay). Elementwise over
 * n parameters, in one pass over memory:
 *   g = grad * grad_scale
 *   exp_avg    = beta1 exp_avg    + (1 - beta1) g
 *   exp_avg_sq = beta2 exp_avg_sq + (1 - beta2) g^2
 *   param     -= lr * ( exp_avg / (1 - beta1^step)
 *                       / (sqrt(exp_avg_sq / (1 - beta2^step)) + eps)
 *                       + weight_decay * param )
 *   param_bf16 = bf16(param) (round to nearest even), when non-null.
 * param, exp_avg, exp_avg_sq: fp32 [n], updated in place (caller-owned device
 * memory, 16-byte aligned); grad fp32 [n] (16-byte aligned); param_bf16 [n]
 * bf16 (8-byte aligned) or NULL. The layout is the caller's: the flat buffer of
 * a layer's six adapter tensors in the order dA[0..2], dB[0..2] lets one call
 * update a whole layer. step >= 1; 0 <= beta1, beta2 < 1; eps > 0; lr,
 * weight_decay >= 0 (else TQP_ERR_INVALID_ARG). A non-finite gradient raises
 * TQP_STATUS_NONFINITE.
 * ------------------------------------------------------------------------- */
int tqp_adamw_step(float* param, float* exp_avg, float* exp_avg_sq, const float* grad, uint16_t* param_bf16, size_t n,
                   float lr, float beta1, float beta2, float eps, float weight_decay, int step, float grad_scale,
                   int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * tqp_debug_set_wait_limit_ns: test hook for the failure path, not for normal
 * use. Every device-side barrier wait in the library's kernels is bounded; this
 * sets that bound for the launches that follow in this process (0 restores the
 * default of 2 s). A wait that runs out sets TQP_STATUS_TIMEOUT, every role of
 * the CTA leaves its loop, copies and MMAs in flight are drained, and the call
 * returns with undefined outputs; the CUDA context stays usable. A limit far
 * below the kernels' normal waits (say 1 ns) makes the next launch time out on
 * purpose. Process-wide; not synchronised with launches on other threads.
 * Returns TQP_OK.
 * ------------------------------------------------------------------------- */
int tqp_debug_set_wait_limit_ns(unsigned long long ns);

#ifdef __cplusplus
}
#endif

#endif /* TQP_MOE_H_ */
