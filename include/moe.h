/*
 * moe.h - C ABI of the B200 (sm_100a) Kimi-K3 MoE feed-forward layer.
 *
 * The layer (what the source pages fix):
 *   - "Kimi K3.1 Pro vs gpt-oss-120b" (archdiff), component table, rows "Sigmoid router
 *     with Quantile Balancing", "Stable LatentMoE routed experts (SiTU-GLU)" and
 *     "Shared expert": sigmoid scores pick 16 of 896 GLU experts per token; one always-on,
 *     ungated bf16 shared expert reads the same input; the block diagram adds the two.
 *   - "Kimi K3" (llm-atlas), raw config fields: hidden_size 7168, num_experts 896,
 *     num_experts_per_token 16, moe_intermediate_size 3072, moe_renormalize true,
 *     routed_scaling_factor 1; Key facts, Dtype row: experts MXFP4, shared expert high
 *     precision.
 *   - "Kimi K3, previewed" (embedl blog), specifications figure caption: MXFP4 weights,
 *     MXFP8 activations.
 * Readings where the pages are silent: the GLU activation is SiLU (the SiTU formula is
 * unpublished), experts act on d_model directly, the router bias is added to the logit,
 * ties in top-k go to the lower expert index, the GLU output is requantised to MXFP8
 * before the down projection.
 *
 * Conventions for every call:
 *   - Pointers marked "device" are CUDA device pointers owned by the caller; the library
 *     never frees them.  "host" pointers are ordinary CPU memory.
 *   - Matrices are row-major.  Weights are stored out x in (row = output channel).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*, NULL = legacy
 *     default stream); none synchronises the host except moe_plan_check and
 *     moe_plan_stage_ms.  The layer's kernels are launched with programmatic stream
 *     serialization: each may start its prologue while the previous kernel on the stream
 *     finishes, but touches no global memory before that kernel has completed, so stream
 *     order holds for the caller's work before and after as usual.
 *   - Errors are returned as moe_status_t; nothing is thrown.  Argument checks happen
 *     before any launch, so an error return leaves outputs untouched.
 *   - Device-side faults (an out-of-range expert id, a pipeline wait that timed out) are
 *     OR-ed into the plan's status word; moe_plan_check reads and clears it.
 */
#ifndef MOE_SM100_H
#define MOE_SM100_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_plan_s* moe_plan_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum value */
  MOE_ERR_UNSUPPORTED_SHAPE = 2, /* d, I, I_shared not multiples of 128; k > 32; T > T_max */
  MOE_ERR_ALIGNMENT = 3,         /* a pointer below its required alignment */
  MOE_ERR_CUDA = 4,              /* a CUDA runtime / driver call or launch failed */
  MOE_ERR_TIMEOUT = 5,           /* a kernel gave up on a bounded wait (moe_plan_check) */
  MOE_ERR_NOT_INITIALIZED = 6,   /* no workspace attached to the plan */
  MOE_ERR_DEVICE_FAULT = 7       /* a kernel flagged bad input (e.g. expert id >= E) */
} moe_status_t;

/* GLU activation of every expert of the layer, routed and shared: a = glu(g, u) with
 * g = x Wg^T, u = x Wu^T.
 *   MOE_ACT_SILU_GLU (default; the pages name SiTU-GLU but publish no formula):
 *     a = g / (1 + exp(-g)) * u.
 *   MOE_ACT_CLAMPED_SWIGLU: the gpt-oss expert of "Kimi K3.1 Pro vs gpt-oss-120b"
 *     (archdiff), component table, routed-experts row.  g_c = min(g, 7),
 *     u_c = clamp(u, -7, 7), a = (u_c + 1) * g_c / (1 + exp(-1.702 g_c)). */
typedef enum { MOE_ACT_SILU_GLU = 0, MOE_ACT_CLAMPED_SWIGLU = 1 } moe_act_t;
/* Router bias.
 *   MOE_BIAS_LOGIT (default): z = x.W_r + b; selection and weights both come from z.
 *   MOE_BIAS_SELECT_ONLY: the per-expert "selection bias" of the router row in the same
 *     table, with topk_method noaux_tc from the raw config of "Kimi K3" (llm-atlas).
 *     Experts are chosen by z + b, computed in fp32, with the same tie rule.  The weights
 *     come from the unbiased s = sigmoid(z), and logits_opt receives z without b. */
typedef enum { MOE_BIAS_LOGIT = 0, MOE_BIAS_SELECT_ONLY = 1 } moe_bias_mode_t;

/* Packed MXFP4 expert weights (device pointers, all 256-byte aligned).
 *   Rows of gate and up are channel blocks of 128 interleaved as gate[0:128], up[0:128],
 *   gate[128:256], up[128:256], ... (2I packed rows); down has d rows (output channels).
 *   w_gu: E2M1 codes, tile-major [E][2I/256][d/128][256 rows][64 B]: 128 consecutive input
 *         elements of a packed row per 64 bytes, element 2j in the low nibble of byte j.
 *   s_gu: E8M0 scales (one per 32 input elements) in the tensor-core scale-factor tiling
 *         [E][2I/256][d/128][2][512]: packed row r of a 256-row tile, 32-block b of the
 *         K tile -> half r/128, byte (r%32)*16 + ((r%128)/32)*4 + b.
 *   w_dn: E2M1 codes of down, [E][ceil(d/256)][I/128][256][64 B] (rows past d are zero).
 *   s_dn: E8M0 scales of down, [E][ceil(d/256)][I/128][2][512].
 * Sizes come from moe_expert_bytes; contents from moe_pack_expert_mxfp4. */
typedef struct {
  void* w_gu;
  void* s_gu;
  void* w_dn;
  void* s_dn;
} moe_experts_mxfp4;

/* bf16 shared expert (device pointers, 16-byte aligned).
 *   w_gu: [2 I_s][d], gate/up interleaved in 128-row blocks as above.
 *   w_dn: [d][I_s]. */
typedef struct {
  void* w_gu;
  void* w_dn;
} moe_shared_bf16;

/* ---- plan ---------------------------------------------------------------------------
 * moe_plan_create: checks the layer shape and the device, allocates nothing on the
 * device.  T_max bounds the tokens of any later call; d, I, I_shared multiples of 128
 * (I_shared = 0: no shared expert); 1 <= k <= min(E, 32); E <= 4096.
 * flags: 0 or MOE_FLAG_STATIC_ROUTER.  With it, moe_route splits W_r into its three bf16
 * terms only when W_r is a different pointer from the one it split last (or on the first
 * call) and reuses them otherwise.  The caller then must not change the contents behind
 * an unchanged pointer; inference weights qualify.  Without it, every call splits again
 * (E*d*4 bytes in, E*d*6 out).  Any other bit is MOE_ERR_INVALID_ARG.
 * Returns the plan in *out (host object, freed by moe_plan_destroy). */
enum { MOE_FLAG_STATIC_ROUTER = 1 };
moe_status_t moe_plan_create(int T_max, int d, int E, int k, int I, int I_shared,
                             moe_act_t act, moe_bias_mode_t bias_mode, int flags,
                             moe_plan_t* out);
/* Device workspace the plan needs for T_max tokens, in bytes (host output). */
moe_status_t moe_plan_workspace_bytes(moe_plan_t plan, size_t* bytes);
/* Attach caller-owned device workspace (256-byte aligned, >= moe_plan_workspace_bytes).
 * The plan borrows it until destroyed or given another one. */
moe_status_t moe_plan_set_workspace(moe_plan_t plan, void* dev_ptr, size_t bytes);
/* Synchronises `stream`, returns MOE_ERR_TIMEOUT / MOE_ERR_DEVICE_FAULT if a kernel since
 * the last check flagged one (bit values in *device_bits, may be NULL), and clears it. */
moe_status_t moe_plan_check(moe_plan_t plan, void* stream, unsigned int* device_bits);
moe_status_t moe_plan_destroy(moe_plan_t plan);
const char* moe_status_string(moe_status_t s);

/* ---- a1: MXFP8 activation quantiser ------------------------------------------------
 * OCP MX rule per 32-element block along a row: scale byte = floor(log2 amax) - 8 + 127
 * (clamped to [0, 254]; all-zero block -> 0), element = E4M3 round-to-nearest-even of
 * v / 2^(scale-127), saturating to +-448, sign kept.
 * x_bf16: device [rows][cols] bf16; q_e4m3: device [rows][cols]; scale_e8m0: device
 * [rows][cols/32].  cols % 32 == 0; x 16-byte aligned, q 16-byte aligned. */
moe_status_t moe_quant_mxfp8(const void* x_bf16, int rows, int cols, uint8_t* q_e4m3,
                             uint8_t* scale_e8m0, void* stream);

/* ---- a2/a3: router --------------------------------------------------------------------
 * Source: "Kimi K3.1 Pro vs gpt-oss-120b" (archdiff), component table, row "Sigmoid router
 * with Quantile Balancing" (sigmoid scores pick 16 of 896 experts); "Kimi K3" (llm-atlas),
 * raw config fields moe_router_activation_func sigmoid, num_experts_per_token 16,
 * moe_renormalize true, routed_scaling_factor 1.
 * z = x . W_r + bias (fp32-accurate: W_r is split into three bf16 terms on the tensor
 * cores), s = sigmoid(z); per token the k largest z in descending order (lower expert
 * index on ties) and w_j = s_j / sum of the selected s.  With MOE_BIAS_SELECT_ONLY the
 * bias enters only the selection key z + b (see moe_bias_mode_t).  Two kernels (plus the
 * fp32 -> three-plane split of W_r, see MOE_FLAG_STATIC_ROUTER): the logit GEMM, then a
 * selection kernel that sums the GEMM's K-split partials (when it split K) and selects
 * in two stages inside each CTA: 8 warps each list a token's k best keys in one eighth
 * of the experts, and one warp merges the 8 lists.
 * x_bf16: device [T][d]; W_r: device fp32 [d][E]; bias: device fp32 [E] or NULL;
 * idx: device int32 [T][k]; w: device fp32 [T][k]; logits_opt: device fp32 [T][E] or
 * NULL (receives z).  Uses the plan workspace. */
moe_status_t moe_route(moe_plan_t plan, const void* x_bf16, int T, const float* W_r,
                       const float* bias, int32_t* idx, float* w, float* logits_opt,
                       void* stream);

/* ---- Quantile Balancing inputs and hook ----------------------------------------------
 * Source: "Kimi K3.1 Pro vs gpt-oss-120b" and "Gemma 4 31B vs Kimi K3" (archdiff),
 * component tables, router row: each expert's selection bias is set every step from a
 * quantile of routing margins; "Kimi K3, previewed" (embedl blog), "Stable LatentMoE"
 * section: allocation derived from router-score quantiles.  The update rule itself is not
 * published, so the library computes what such a rule reads and hands it to the caller's.
 * Reading: the routing margin of expert e for token t is m[t][e] = key[t][e] - key_(k)(t),
 * the expert's selection key minus the token's k-th largest key (the top-k threshold;
 * selected experts have m >= 0), key = z or, with a select-only bias, z + b, all in fp32.
 * The level-q quantile of expert e is the order statistic of rank clamp(ceil(q T), 1, T)
 * (1-based, ascending) of m[0..T)[e], rank computed in double on the host.
 *
 * moe_route_margin_quantiles: logits: device fp32 [T][E] (moe_route's logits_opt, i.e. z
 * without a select-only bias); select_bias: device fp32 [E] or NULL (NULL: key = z);
 * levels: host double [n_levels], each in [0, 1]; quantiles: device fp32 [n_levels][E],
 * row i for levels[i].  1 <= n_levels <= 16, 1 <= T <= T_max.  Exact (selection, no
 * interpolation).  Two kernels on `stream`, no host synchronisation; uses the plan's
 * workspace (the k-th keys), so calls on one plan are ordered on one stream. */
moe_status_t moe_route_margin_quantiles(moe_plan_t plan, const float* logits, const float* select_bias,
                                        int T, const double* levels, int n_levels, float* quantiles,
                                        void* stream);
/* The caller's bias-update rule.  Called on the calling host thread, after the quantile
 * kernels were enqueued on `stream` (and before they ran): it must enqueue its own device
 * work on that stream.  quantiles: device fp32 [n_levels][E] (plan workspace, valid until
 * the next call on the plan); bias: device fp32 [E], the bias of this step; bias_next:
 * device fp32 [E] to receive the next step's bias; user: passed through. */
typedef void (*moe_bias_rule_t)(const float* quantiles, int n_levels, int E, const float* bias,
                                float* bias_next, void* stream, void* user);
/* moe_quantile_balance: margin quantiles of this step's routing, then rule(...).  The key
 * is z + bias under MOE_BIAS_SELECT_ONLY and z under MOE_BIAS_LOGIT (the bias is already in
 * z); logits as for moe_route_margin_quantiles.  The rule is the caller's: the library
 * does no arithmetic on the bias itself. */
moe_status_t moe_quantile_balance(moe_plan_t plan, const float* logits, const float* bias, int T,
                                  const double* levels, int n_levels, moe_bias_rule_t rule, void* user,
                                  float* bias_next, void* stream);

/* ---- a4: grouping by expert -----------------------------------------------------------
 * counts[e] = assignments to expert e; offsets = exclusive prefix sum (offsets[E] = T*k);
 * perm_tok[p] = token of the p-th assignment in (expert, token) order; inv[t][j] = the
 * position of assignment (t, j).  idx: device int32 [T][k] with distinct ids per token.
 * Outputs are device int32 arrays of E, E+1, T*k, T*k entries.  Ids outside [0, E) are
 * skipped and flagged (MOE_ERR_DEVICE_FAULT at moe_plan_check). */
moe_status_t moe_permute(moe_plan_t plan, const int32_t* idx, int T, int32_t* counts,
                         int32_t* offsets, int32_t* perm_tok, int32_t* inv, void* stream);

/* ---- a4 without device allocation ---------------------------------------------------
 * The same grouping as moe_permute, for callers that cannot call cudaMalloc: code that
 * runs inside a host application or serving engine which owns the whole device-memory
 * budget (and may forbid or account every allocation), or a thread that must not take the
 * allocator's locks or risk the implicit device synchronisation of cudaMalloc/cudaFree.
 * It needs no plan and no workspace.  The source pages have no counterpart; this is a
 * deployment aid of this library.
 * Scratch: a fixed 256 KiB array in the library's device memory, held by every GPU that
 * loads the library until the process exits.  Calls are rejected with
 * MOE_ERR_UNSUPPORTED_SHAPE when 256 + ceil(T/256)*E*4 (rounded up to 256) + (E+1)*4
 * bytes exceed it (e.g. T <= 18432 at E = 896).  All calls share the array, so two calls
 * whose work overlaps on the GPU (different streams, or different host threads) race.
 * The first call on a device looks up the array's device address (with that device
 * current) and caches it per device and CUDA context (a new context, e.g. after
 * cudaDeviceReset, gets a fresh lookup); make that first call before any stream capture.
 * Arguments and outputs as moe_permute (device pointers, caller-owned); ids outside
 * [0, E) are skipped and leave inv = -1 (no status is reported). */
moe_status_t moe_permute_noalloc(const int32_t* idx, int T, int E, int k, int32_t* counts,
                                 int32_t* offsets, int32_t* perm_tok, int32_t* inv,
                                 void* stream);

/* ---- a4..a9: the layer ----------------------------------------------------------------
 * Source: "Kimi K3.1 Pro vs gpt-oss-120b" (archdiff), component table, rows "Stable
 * LatentMoE routed experts (SiTU-GLU)" and "Shared expert", and its block diagram, which
 * adds the routed and shared outputs; "Kimi K3" (llm-atlas), Key facts, Dtype row (MXFP4
 * experts, high-precision shared expert); "Kimi K3, previewed" (embedl blog),
 * specifications figure caption (MXFP4 weights, MXFP8 activations).
 * y = bf16( shared(x) + sum_j w[t][j] * expert_{idx[t][j]}(x) ), where an expert is
 * down(glu(x Wg^T, x Wu^T)) on MXFP8 x and MXFP4 weights, its GLU output requantised
 * to MXFP8, and shared(x) = bf16(glu(x Wsg^T, x Wsu^T)) Wsd^T in bf16/fp32 (glu: the
 * plan's moe_act_t).
 * x_bf16: device [T][d]; idx/w: device [T][k] (e.g. from moe_route); experts: packed
 * weights; shared: NULL when the plan has I_shared = 0; y_bf16: device [T][d].
 * T = 0 is a no-op.  Uses the plan workspace (one call at a time per plan). */
moe_status_t moe_forward(moe_plan_t plan, const void* x_bf16, int T, const int32_t* idx,
                         const float* w, const moe_experts_mxfp4* experts,
                         const moe_shared_bf16* shared, void* y_bf16, void* stream);

/* ---- latent option ---------------------------------------------------------------------
 * Reading of the pages' "Stable LatentMoE": the routed experts run on a d_latent-wide
 * latent with an RMSNorm before them ("Kimi K3.1 Pro vs gpt-oss-120b" and "Gemma 4 31B vs
 * Kimi K3", component tables, routed-experts row; "Kimi K3" (llm-atlas), raw config:
 * routed_expert_hidden_size 3584, latent_moe_use_norm, rms_norm_eps 1e-5).  The pages do
 * not publish where the projections sit, so this is the plainest reading:
 *   x_l = x W_ld^T (bf16 x bf16, fp32 accumulation)
 *   x_n = bf16(x_l / sqrt(mean(x_l^2) + eps) * gamma)
 *   y_l = bf16(sum_j w[t][j] * expert_{idx[t][j]}(x_n))   (experts packed with d = d_latent)
 *   y   = bf16(y_l W_lu^T + shared(x))                    (fp32 sum; shared reads x itself)
 * moe_plan_set_latent: d_latent % 128 == 0 and 0 < d_latent <= d; eps > 0.  Call it before
 * moe_plan_workspace_bytes / moe_plan_set_workspace (the workspace grows by the latent
 * buffers); MOE_ERR_INVALID_ARG once a workspace is attached. */
typedef struct {
  const void* w_down;   /* bf16 [d_latent][d]: x -> latent (device) */
  const float* gamma;   /* fp32 [d_latent]: RMSNorm gain (device) */
  const void* w_up;     /* bf16 [d][d_latent]: latent -> d (device) */
} moe_latent_bf16;
moe_status_t moe_plan_set_latent(moe_plan_t plan, int d_latent, float eps);
/* The layer with the latent option; arguments as moe_forward plus `latent`.  The plan
 * must have had moe_plan_set_latent; experts are packed with d = d_latent. */
moe_status_t moe_forward_latent(moe_plan_t plan, const void* x_bf16, int T, const int32_t* idx,
                                const float* w, const moe_latent_bf16* latent,
                                const moe_experts_mxfp4* experts, const moe_shared_bf16* shared,
                                void* y_bf16, void* stream);

/* ---- setup helpers (not on the timed path) --------------------------------------------
 * Byte sizes of the four packed expert arrays for E experts (host outputs). */
moe_status_t moe_expert_bytes(int d, int I, int E, size_t* w_gu, size_t* s_gu, size_t* w_dn,
                              size_t* s_dn);
/* MXFP4-quantise expert e's fp32 masters (device: w_gate, w_up [I][d], w_down [d][I];
 * blocks of 32 along the input dimension, same MX rule as above with E2M1 elements,
 * max 6, emax 2) into the packed arrays of `dst`. */
moe_status_t moe_pack_expert_mxfp4(int d, int I, int e, const float* w_gate, const float* w_up,
                                   const float* w_down, const moe_experts_mxfp4* dst,
                                   void* stream);
/* Lay out the bf16 shared expert (device: w_gate, w_up [I_s][d], w_down [d][I_s]) into
 * dst (device buffers of 2*I_s*d and d*I_s bf16). */
moe_status_t moe_pack_shared_bf16(int d, int I_shared, const void* w_gate, const void* w_up,
                                  const void* w_down, const moe_shared_bf16* dst, void* stream);

/* ---- tuning options ----------------------------------------------------------------
 * MOE_OPT_PREFETCH_DIST: the routed grouped GEMMs prefetch their weight tiles into L2
 *   this many K tiles ahead of the shared-memory loads (0..64, 0 = off).
 * MOE_OPT_PREFETCH_B: accepted and ignored (reserved).
 * MOE_OPT_TILE_N: token rows per routed grouped-GEMM tile.  0 (default) picks per call:
 *   32 rows (6-stage pipeline) when T*k <= 8*E, i.e. a few tokens per expert and a pure
 *   weight stream, else 176 rows (4 stages); both put 256 weight rows on the MMA's M side
 *   and the token rows on its N side.  128 selects the other orientation: token rows on M
 *   (up to 128 per tile) and 256 weight rows on N.  160 selects tiles of up to 160 token
 *   rows run on clusters of two CTAs (one MMA spans two SMs: each holds its own 256 weight
 *   rows and half of the token rows; five pipeline stages); a GEMM whose weight rows do not
 *   form an even number of 256-row tiles runs its 160-row tiles on single CTAs instead.
 *   32, 128, 160 or 176 forces one configuration; any other value is MOE_ERR_INVALID_ARG.
 *   The dense shared-expert GEMMs use 32-row tiles when T*k <= 8*E and 176 otherwise.  The
 *   K loop runs in the same order in all of them, and the tensor core accumulates a row the
 *   same way in either orientation and on one or two SMs: results are identical.
 * MOE_OPT_ROUTER_SPLIT (read only): the number of K splits the last moe_route used for
 *   the router GEMM (1 = none).  With few tokens the router splits d over up to one
 *   CTA per SM; each split stores its fp32 partial, and the selection kernel that follows
 *   adds the partials in split order (plus the bias) before it selects.
 * MOE_OPT_SHARED_SPLIT / MOE_OPT_SHARED_SPLIT_DOWN (read only): K splits of the shared
 *   expert's gate/up and down GEMMs in the last moe_forward (1 = none; 0 without a shared
 *   expert).  With few tokens these dense GEMMs split K over the SMs.  Each split GEMM writes
 *   fp32 partials, and one more kernel adds them in split order (the gate/up one also applies
 *   the GLU), so each split adds one launch.
 * moe_plan_get_option reads an option back (host int); for MOE_OPT_TILE_N it returns the
 * tile rows that the last moe_forward on this plan used (0 before the first call), which
 * fixes the tile-major layout of the token-side scale blocks (debug buffers 1 and 3). */
enum { MOE_OPT_PREFETCH_DIST = 0, MOE_OPT_PREFETCH_B = 1, MOE_OPT_TILE_N = 2, MOE_OPT_ROUTER_SPLIT = 3,
       MOE_OPT_SHARED_SPLIT = 4, MOE_OPT_SHARED_SPLIT_DOWN = 5 };
moe_status_t moe_plan_set_option(moe_plan_t plan, int option, int value);
moe_status_t moe_plan_get_option(moe_plan_t plan, int option, int* value);

/* ---- per-stage timing ---------------------------------------------------------------
 * With profiling on, every stage of moe_route / moe_forward is bracketed by two CUDA
 * events recorded on the call's stream (no host synchronisation).  moe_plan_stage_ms
 * synchronises on them and returns, per stage, the summed elapsed milliseconds and the
 * number of recorded launches since profiling was enabled or last queried (host arrays of
 * n >= MOE_NUM_STAGES entries; `launches` may be NULL), then forgets them. */
enum {
  MOE_STAGE_ROUTER_SPLIT = 0,    /* W_r -> three bf16 planes */
  MOE_STAGE_ROUTER_GEMM = 1,     /* logits on the tensor cores (fp32 partials when K is split) */
  MOE_STAGE_TOPK = 2,            /* split sum + bias, top-k selection, sigmoid weights */
  MOE_STAGE_PERMUTE = 3,         /* histogram, scan, placement (3 kernels) */
  MOE_STAGE_QUANT = 4,           /* MXFP8 quantise + scatter to expert order */
  MOE_STAGE_GATE_UP = 5,         /* routed gate/up GEMM + GLU + MXFP8 requant */
  MOE_STAGE_DOWN = 6,            /* routed down GEMM */
  MOE_STAGE_SHARED_GATE_UP = 7,  /* shared expert gate/up + GLU */
  MOE_STAGE_SHARED_DOWN = 8,     /* shared expert down */
  MOE_STAGE_COMBINE = 9,         /* weighted combine */
  MOE_STAGE_LATENT_IN = 10,      /* latent option: x -> latent GEMM + RMSNorm (2 kernels) */
  MOE_STAGE_LATENT_OUT = 11,     /* latent option: latent -> d GEMM + final add (2 kernels) */
  MOE_NUM_STAGES = 12
};
moe_status_t moe_plan_set_profiling(moe_plan_t plan, int enable);
moe_status_t moe_plan_stage_ms(moe_plan_t plan, float* ms, int* launches, int n);

/* ---- introspection (tests) ----------------------------------------------------------
 * Device pointer and size of a workspace buffer after a call, for checking the steps:
 *   0 xq  E4M3 [T*k][d] activations in expert order
 *   1 xs  scales of xq, tile-major: for group-tile g (tiles of <= 176 rows per expert,
 *         ceil(count/176) tiles of round16(ceil(count/tiles)) rows each, numbered in
 *         expert order) and 128-column K tile kt, 1 KB at (g*(d/128) + kt)*1024; row n of
 *         the tile, 32-block j of the K tile at (n/128)*512 + (n%32)*16 + ((n%128)/32)*4 + j
 *   2 hq  E4M3 [T*k][I] GLU output in expert order
 *   3 hs  scales of hq, same tile-major layout with I/128 K tiles
 *   4 O   bf16 [T*k][d] expert outputs in expert order
 *   5 ys  fp32 [T][d] shared expert output
 *   6 logits fp32 [T][E]
 *   7 quantiles fp32 [16][E]: the buffer moe_quantile_balance hands to the bias rule
 * Row counts use the T of the last call. */
moe_status_t moe_debug_buffer(moe_plan_t plan, int which, void** dev_ptr, size_t* bytes);

/* ---- failure-path probe -----------------------------------------------------------------
 * Launches one CTA on `stream` that waits, with the same bounded mbarrier wait the GEMM
 * and router kernels use, on a barrier that nothing ever arrives at.  After the wait's
 * limit (1 s of %globaltimer) the kernel records MOE_ERR_TIMEOUT in the plan's status word
 * and returns.  The context stays usable, and the next moe_plan_check reports
 * MOE_ERR_TIMEOUT and clears it.  It tests the timeout path without faulting or hanging
 * the GPU.  Needs the plan's workspace. */
moe_status_t moe_debug_timeout_probe(moe_plan_t plan, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_SM100_H */
