/*
 * rtvla.h — C ABI of librtvla.so: the π0.5 action-expert flow-matching denoise loop, the
 * Gemma-2B-shaped prefix pass that fills its KV cache, and the image front-end (SigLIP tower +
 * projector) that produces the prefix's image embeddings, as hand-written CUDA for sm_100a.
 *
 * What the calls compute is defined by:
 *   [BLOG]  Realtime-VLA tech blog (blog.w4k4.me): "pi0.5 inference flow" (encoder phase run
 *           once, then a 10-step denoise loop), "Inference branch structure" (encoder-only
 *           and decoder-only branches of PaliGemmaWithExpertModel.forward), "Per-layer
 *           processing (PiGemmaDecoderLayer.forward)", "Precompute (__init__)", "CUDA Graph"
 *           (inputs copied in, one replay) and "Static buffers".
 *   [PAPER] "Running VLAs at Real-time Speed" (arXiv 2510.26742), Sec. 3.1-3.2, Table 1.
 *
 * Conventions for every call:
 *   - All tensors are row-major and contiguous.  Weight matrices use the (out, in) layout of
 *     a Linear layer: element [o][i] multiplies input i into output o.  "bf16" is IEEE
 *     bfloat16 (uint16 storage); "f32" is IEEE float.
 *   - Pointers named *device* must point to memory of the CUDA device that was current when
 *     rtvla_create ran; pointers named *host* are ordinary CPU memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Work is
 *     enqueued asynchronously unless the call says otherwise.
 *   - Argument and shape errors are returned synchronously, before anything is enqueued.
 *     Errors the GPU detects (a bounded wait that expired, an index out of range, a pad mask
 *     that is not a prefix) set a device error word that rtvla_sync_status reports.  Nothing
 *     aborts, traps or throws across the ABI.
 *   - One context serves one stream at a time: calls on one context must not overlap on the
 *     GPU (they share the context's static activation buffers).
 */
#ifndef RTVLA_H
#define RTVLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct rtvla_ctx rtvla_ctx; /* opaque; owned by the library */

typedef enum {
  RTVLA_OK = 0,
  RTVLA_ERR_INVALID_ARG = 1,     /* null pointer, negative size, bad enum value */
  RTVLA_ERR_SHAPE = 2,           /* batch / prefix length / chunk beyond the context's capacity */
  RTVLA_ERR_MASK_NOT_PREFIX = 3, /* pad mask has a valid token after a padded one (device-detected) */
  RTVLA_ERR_OOM = 4,             /* cudaMalloc failed while creating the context */
  RTVLA_ERR_CUDA = 5,            /* a CUDA runtime call failed; the context may be unusable */
  RTVLA_ERR_DEVICE_TIMEOUT = 6,  /* a bounded device-side wait expired (device-detected) */
  RTVLA_ERR_UNSUPPORTED = 7,     /* model shape the kernels are not built for */
  RTVLA_ERR_DEVICE_BOUNDS = 8,   /* a valid length exceeded its buffer (device-detected, clamped) */
  RTVLA_ERR_GUARD_OVERWRITE = 9  /* checked mode: a guard band around a library buffer changed */
} rtvla_status;

/* Engines that run the denoise loop (rtvla_config.engine).  The persistent engine applies to
 * calls with batch 1 and chunk <= 64 on a GPU where its cooperative launch fits (one CTA of
 * 320 threads and ~218 KB of shared memory per SM, >= 64 SMs; rtvla_kernels_per_call then
 * returns 1).  Results of the two engines agree within the parity tolerance, not bitwise
 * (split-K sums are reduced in a different order). */
enum {
  RTVLA_ENGINE_AUTO = 0,       /* the persistent kernel when it applies, else layered */
  RTVLA_ENGINE_LAYERED = 1,    /* one kernel per phase, the whole loop captured as one CUDA graph */
  RTVLA_ENGINE_PERSISTENT = 2  /* one persistent kernel per call; calls it cannot serve return
                                  RTVLA_ERR_UNSUPPORTED */
};

/* Model variants (rtvla_config.variant).  [PAPER] Sec. 1.1.2 and the "Running VLAs at
 * Real-time Speed" summary ("How": the action time encoder): π0 routes the robot state and
 * the noisy actions to the action expert; π0.5 conditions the expert on the time through
 * AdaRMS [BLOG "pi0.5 inference flow"]. */
enum {
  RTVLA_VARIANT_PI05 = 0, /* AdaRMS (scale, shift, gate) from the time MLP; gated residuals */
  RTVLA_VARIANT_PI0 = 1   /* suffix = [state token ; actions]; action tokens from the action-time
                             MLP; plain RMSNorm (scale 1 + w); ungated residuals; final norm.
                             Both engines; the persistent one needs chunk + 1 <= 64 */
};

/*
 * Model and capacity description.  The kernels are built for the π0.5 shapes of [BLOG
 * "pi0.5 inference flow"]: width 1024, MLP 4096, 8 query heads x 256, 1 KV head, action
 * dim 32 (expert); width 2048, MLP 16384, 8 x 256, 1 KV head (prefix pass).  Other values
 * return RTVLA_ERR_UNSUPPORTED.  n_layers and n_steps are free (1..64 and 1..64).
 */
typedef struct {
  int n_layers;    /* expert layers L (18; 2 for the tiny expert); the prefix pass has as many */
  int width;       /* D = 1024 */
  int mlp_dim;     /* F = 4096 */
  int n_q_heads;   /* 8 */
  int n_kv_heads;  /* 1 */
  int head_dim;    /* 256 */
  int action_dim;  /* 32 */
  int chunk;       /* C, actions per chunk (1..256) */
  int n_steps;     /* Euler steps S (10); t_k = 1 - k/S, dt = -1/S */
  int max_prefix;  /* capacity P_max of the prefix KV cache in tokens (>= 1) */
  int max_batch;   /* largest batch any call will use (>= 1) */
  int final_norm;  /* 1: AdaRMS before action_out_proj; 0: none */
  int has_prefill; /* 1: also build the prefix pass (needs the pf_* weights) */
  int pf_width;    /* 2048 when has_prefill */
  int pf_mlp_dim;  /* 16384 when has_prefill */
  int engine;      /* RTVLA_ENGINE_* */
  float rms_eps;   /* 1e-6 */
  float rope_theta;/* 10000 */
  int variant;     /* RTVLA_VARIANT_* (0 = π0.5) */
} rtvla_config;

/*
 * Weights: device pointers to bf16 tensors in (out, in) layout, owned by the caller and
 * read only during rtvla_create (the library keeps its own folded copies, so the caller
 * may free these when rtvla_create returns).  Per-layer fields are host arrays of
 * n_layers device pointers.
 */
typedef struct {
  const void *action_in_w;  /* [D][A]  action_in_proj */
  const void *action_in_b;  /* [D] */
  const void *action_out_w; /* [A][D]  action_out_proj */
  const void *action_out_b; /* [A] */
  const void *time_in_w;    /* [D][D]  time_mlp_in */
  const void *time_in_b;    /* [D] */
  const void *time_out_w;   /* [D][D]  time_mlp_out */
  const void *time_out_b;   /* [D] */
  const void *const *wq;    /* [L] -> [H*hd][D] */
  const void *const *wk;    /* [L] -> [hd][D] */
  const void *const *wv;    /* [L] -> [hd][D] */
  const void *const *wo;    /* [L] -> [D][H*hd] */
  const void *const *wg;    /* [L] -> [F][D]  gate_proj */
  const void *const *wu;    /* [L] -> [F][D]  up_proj */
  const void *const *wd;    /* [L] -> [D][F]  down_proj */
  const void *const *ada_attn_w; /* [L] -> [3D][D]  input_layernorm dense (scale|shift|gate) */
  const void *const *ada_attn_b; /* [L] -> [3D] */
  const void *const *ada_ffn_w;  /* [L] -> [3D][D]  post_attention_layernorm dense */
  const void *const *ada_ffn_b;  /* [L] -> [3D] */
  const void *ada_final_w;  /* [3D][D]  final norm dense (used when final_norm = 1) */
  const void *ada_final_b;  /* [3D] */
  /* prefix pass (has_prefill = 1): Gemma RMSNorm weights w (scale 1 + w) and projections */
  const void *const *pf_ln1; /* [L] -> [Dp] */
  const void *const *pf_wq;  /* [L] -> [H*hd][Dp] */
  const void *const *pf_wk;  /* [L] -> [hd][Dp] */
  const void *const *pf_wv;  /* [L] -> [hd][Dp] */
  const void *const *pf_wo;  /* [L] -> [Dp][H*hd] */
  const void *const *pf_ln2; /* [L] -> [Dp] */
  const void *const *pf_wg;  /* [L] -> [Fp][Dp] */
  const void *const *pf_wu;  /* [L] -> [Fp][Dp] */
  const void *const *pf_wd;  /* [L] -> [Dp][Fp] */
  /* π0 (variant RTVLA_VARIANT_PI0; then time_in_*, ada_* are not read, action_in_* and
   * action_out_* are) */
  const void *state_w;           /* [D][A]   state_proj */
  const void *state_b;           /* [D] */
  const void *action_time_in_w;  /* [D][2D]  action_time_mlp_in over [action_in_proj(x) ; SinEmb(t)] */
  const void *action_time_in_b;  /* [D] */
  const void *action_time_out_w; /* [D][D]   action_time_mlp_out */
  const void *action_time_out_b; /* [D] */
  const void *const *ln1;        /* [L] -> [D]  input_layernorm weight w (scale 1 + w) */
  const void *const *ln2;        /* [L] -> [D]  post_attention_layernorm weight w */
  const void *final_ln;          /* [D]        final norm weight w */
} rtvla_weights;

/*
 * Prefix KV cache (caller-owned device memory).  [BLOG "pi0.5 inference flow", encoder
 * step 4: past_key_values of every layer].  K is stored after RoPE ("rotate half" pairs
 * (d, d+128), position p of prefix token p).  Only tokens [0, valid_len[b]) of sample b are
 * read; the rest may hold anything.
 */
typedef struct {
  void *k;             /* device bf16 [n_layers][batch][prefix_cap][head_dim] */
  void *v;             /* device bf16 [n_layers][batch][prefix_cap][head_dim] */
  int32_t *valid_len;  /* device int32 [batch], each in [0, prefix_cap] */
  int batch;           /* 1..max_batch */
  int prefix_cap;      /* 1..max_prefix, the token stride of k and v */
} rtvla_kv;

/*
 * Creates a context: repacks and folds the weights and builds the per-step tables of
 * [BLOG "Precompute (__init__)"] — time embedding and time MLP for the S fixed timesteps,
 * every AdaRMS dense output (scale, shift, gate) for every (step, layer), Q/K/V
 * concatenated, dt folded into action_out_proj, RoPE cos/sin — and allocates every
 * activation buffer once [BLOG "Static buffers"].  Synchronous.  On success *out owns
 * device memory until rtvla_destroy.  Errors: INVALID_ARG, UNSUPPORTED, OOM, CUDA.
 * Environment read here: RTVLA_WAIT_TIMEOUT_US (bound on every device wait, default
 * 2,000,000), RTVLA_CHECKED and RTVLA_DEVICE_MEMORY_CAP (see rtvla_sync_status),
 * RTVLA_PHASE_STAMPS=<file> (persistent-kernel phase timestamps, written by rtvla_destroy),
 * RTVLA_PAIR_GEMM=1 (the SM-pair form of the layered GEMM; off by default, measured slower).
 */
rtvla_status rtvla_create(const rtvla_weights *w, const rtvla_config *cfg, rtvla_ctx **out);

/* Bytes of K plus V for a cache of `batch` samples x `prefix_cap` tokens (0 on bad args). */
size_t rtvla_kv_bytes(const rtvla_config *cfg, int batch, int prefix_cap);

/*
 * Prefix pass [BLOG "pi0.5 inference flow", encoder steps 3-4; "Inference branch
 * structure", encoder-only branch].  prefix_embeds: device bf16 [batch][prefix_len][pf_width],
 * already scaled by sqrt(2048).  pad_mask: device uint8 [batch][prefix_len], 1 = valid; the
 * valid tokens of each sample must come first.  Fills kv_out->k / kv_out->v for every layer
 * (rows >= the valid length hold unspecified values) and kv_out->valid_len.  The last layer
 * computes K/V only.  Errors: INVALID_ARG, SHAPE (batch > max_batch, prefix_len >
 * kv_out->prefix_cap or > max_prefix), UNSUPPORTED (no prefill built); device-detected
 * MASK_NOT_PREFIX through rtvla_sync_status.
 */
rtvla_status rtvla_prefill(rtvla_ctx *ctx, const void *prefix_embeds, const uint8_t *pad_mask,
                           int batch, int prefix_len, const rtvla_kv *kv_out, void *stream);

/*
 * The denoise loop [BLOG "pi0.5 inference flow", decoder phase steps 1-4; "Inference
 * branch structure", decoder-only branch]: x = noise at t = 1; for k = 0..S-1 the expert
 * predicts v_t from x, the prefix KV and t_k = 1 - k/S, and x += dt * v_t with dt = -1/S.
 * noise, actions_out: device f32 [kv->batch][chunk][action_dim] (may alias).  Runs as one
 * CUDA-graph replay or one persistent launch on `stream`.  Errors: INVALID_ARG, SHAPE;
 * device-detected DEVICE_TIMEOUT / DEVICE_BOUNDS through rtvla_sync_status.
 */
rtvla_status rtvla_sample_actions(rtvla_ctx *ctx, const float *noise, const rtvla_kv *kv,
                                  float *actions_out, void *stream);

/*
 * The π0 denoise loop (context variant RTVLA_VARIANT_PI0) [PAPER summary, "How"; Sec. 1.1.2]:
 * each step builds the suffix [state token ; C action tokens] — state token = state_proj(state);
 * action token = action_time_mlp_out(SiLU(action_time_mlp_in([action_in_proj(x) ; SinEmb(t)]))),
 * computed as SiLU(W_fold x + c_k) with W_fold = action_time_mlp_in[:, :D] @ action_in_proj and
 * the 10 rows c_k tabulated at create time — runs the L layers over those C + 1 tokens
 * (plain RMSNorm, ungated residuals; every suffix token sees every valid prefix key and every
 * suffix token, at positions Lv + i with the state at i = 0), then a final RMSNorm and
 * action_out_proj on the action tokens, and x += dt * v.  noise, actions_out: device f32
 * [batch][chunk][action_dim]; state: device f32 [batch][action_dim].  Errors: INVALID_ARG,
 * SHAPE, UNSUPPORTED (a π0.5 context, or engine PERSISTENT with chunk + 1 > 64 or batch > 1);
 * device-detected errors through rtvla_sync_status.  rtvla_sample_actions on a π0 context returns
 * INVALID_ARG (no state).
 */
rtvla_status rtvla_sample_actions_pi0(rtvla_ctx *ctx, const float *noise, const float *state,
                                      const rtvla_kv *kv, float *actions_out, void *stream);

/*
 * Same loop from host buffers: copies noise (host f32 [batch][chunk][action_dim]), the
 * cache (host bf16 k and v [n_layers][batch][prefix_cap][head_dim], host int32 valid_len
 * [batch]) to the context's device staging, runs the loop, copies the actions back to
 * actions_out (host f32) and waits for the stream.  Host buffers should be pinned for full
 * copy speed.  The staging cache is allocated on first use (RTVLA_ERR_OOM on failure).  A π0
 * context returns RTVLA_ERR_INVALID_ARG (this call carries no state).
 */
rtvla_status rtvla_sample_actions_host(rtvla_ctx *ctx, const float *noise, const void *kv_k,
                                       const void *kv_v, const int32_t *valid_len, int batch,
                                       int prefix_cap, float *actions_out, void *stream);

/*
 * Allocation-free variant of rtvla_sample_actions_host (the paper has no counterpart: this
 * is an integration aid of this library).
 *
 * Who needs it: a robot control loop that runs inference every camera frame must keep a fixed
 * period, and cudaMalloc can block for milliseconds and synchronise the device; some hosts
 * also fix every device-memory budget at start-up.  Such callers create the context once at
 * start-up (rtvla_create allocates) and afterwards may not allocate at all — but
 * rtvla_sample_actions_host allocates its device staging on first use.  This call allocates
 * nothing: it stages the inputs and outputs in one file-scope device array of 32 MiB
 * (RTVLA_STATIC_STAGING_BYTES) that every GPU loading this library holds until the process
 * exits, and it captures no graph.  It runs the engine rtvla_sample_actions would run: the
 * persistent kernel where it applies (batch 1, chunk <= 64, engine AUTO or PERSISTENT);
 * otherwise a layered graph already captured for this shape by rtvla_sample_actions is
 * replayed, and without one the layered kernels are launched directly (slower: one launch
 * per kernel).
 *
 * Arguments, layout and result are those of rtvla_sample_actions_host (host buffers, the
 * call waits for `stream`).  The device of `ctx` must be current.  Errors: INVALID_ARG (also for
 * a π0 context: this call carries no state);
 * SHAPE when batch or prefix_cap exceed the context's capacity or when noise + actions +
 * valid_len + K + V (each rounded up to 256 bytes) need more than 32 MiB, checked before
 * anything is copied; UNSUPPORTED when the engine is PERSISTENT and the call is one it
 * cannot serve; CUDA.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress);
 * make that first call before any stream capture.  All calls share the one array, which
 * keeps the last call's contents (every byte a call reads is written by that call first):
 * calls that overlap on the GPU — from two streams or two contexts on one device — race.
 * The call also writes the context's device argument block, which rtvla_sample_actions and
 * its graphs read: it must not overlap any other sample call on the same context either.
 */
rtvla_status rtvla_sample_actions_host_static(rtvla_ctx *ctx, const float *noise, const void *kv_k,
                                              const void *kv_v, const int32_t *valid_len, int batch,
                                              int prefix_cap, float *actions_out, void *stream);

/*
 * Waits for `stream`, then reads and clears the device error word: RTVLA_OK, or the first
 * device-detected error (DEVICE_TIMEOUT, DEVICE_BOUNDS, MASK_NOT_PREFIX, GUARD_OVERWRITE)
 * since the last call.
 *
 * Checked mode (a run-time race and bounds detector; no counterpart on the pages): with the
 * environment variable RTVLA_CHECKED=1 when rtvla_create runs, every buffer the context
 * allocates sits between two 4096-byte guard bands filled with 0xA5, and this call first
 * enqueues a check of every band on `stream`; a band that changed (a kernel wrote past a
 * buffer) is refilled and reported as RTVLA_ERR_GUARD_OVERWRITE.  A device-memory cap for
 * the context can be set with RTVLA_DEVICE_MEMORY_CAP=<bytes>: rtvla_create then returns
 * RTVLA_ERR_OOM, having freed everything, when the context would need more.
 */
rtvla_status rtvla_sync_status(rtvla_ctx *ctx, void *stream);

/*
 * Test hook of checked mode: overwrites the first byte after the context's residual-stream
 * buffer (the kind of write a kernel that runs one row too far makes), so that the next
 * rtvla_sync_status must report RTVLA_ERR_GUARD_OVERWRITE.  Synchronous.  Errors:
 * INVALID_ARG; UNSUPPORTED when the context is not in checked mode; CUDA.
 */
rtvla_status rtvla_debug_plant_guard_fault(rtvla_ctx *ctx);

/*
 * Test hook: runs the loop with the engine rtvla_sample_actions would run for this call and
 * writes the expert hidden state of step `step` (0-based) before layer 0 and after each
 * layer to h_layers: device f32 [n_layers + 1][batch][chunk][width].  The persistent engine
 * runs the whole loop and records the step on the way; the layered engine stops after it.
 * No actions are written.  Asynchronous.  Errors: INVALID_ARG, SHAPE, UNSUPPORTED (engine
 * PERSISTENT and a call it cannot serve), CUDA.
 */
rtvla_status rtvla_debug_trace(rtvla_ctx *ctx, const float *noise, const rtvla_kv *kv, int step,
                               float *h_layers, void *stream);

/* The test hook of rtvla_debug_trace for a π0 context (state: device f32 [batch][action_dim]);
 * h_layers is device f32 [n_layers + 1][batch][chunk + 1][width], the state token first. */
rtvla_status rtvla_debug_trace_pi0(rtvla_ctx *ctx, const float *noise, const float *state,
                                   const rtvla_kv *kv, int step, float *h_layers, void *stream);

/* Number of kernels of this library one rtvla_sample_actions call launches at `batch`
 * with the context's engine (after the call has been made once at that batch). */
int rtvla_kernels_per_call(rtvla_ctx *ctx, int batch);

/* Selects the engine for later calls (RTVLA_ENGINE_*); INVALID_ARG on a bad value. */
rtvla_status rtvla_set_engine(rtvla_ctx *ctx, int engine);

/* Bounded device waits give up after this many microseconds (default 2,000,000). */
rtvla_status rtvla_set_wait_timeout_us(rtvla_ctx *ctx, long long us);

/* Frees everything the context owns (waits for the device first).  NULL is a no-op. */
void rtvla_destroy(rtvla_ctx *ctx);

/* Static English text for a status code. */
const char *rtvla_status_string(rtvla_status s);

/* =========================================================================================
 * Image front-end: the SigLIP vision tower and the multi_modal_projector, which turn each
 * camera view into the prefix embeddings rtvla_prefill consumes [BLOG "pi0.5 inference
 * flow": model structure (SigLIP, 400M parameters, 224 x 224 image -> 256 tokens), encoder
 * step 1 (256 embeddings per view, scaled by sqrt(2048)) and step 3 (image tokens, then
 * language tokens); class hierarchy (vision_tower: SiglipVisionTransformer, 27 layers;
 * multi_modal_projector: Linear 1152 -> 2048)].  A context of its own, independent of
 * rtvla_ctx; the same conventions (row-major, (out, in) Linear layout, bf16 = IEEE bfloat16,
 * asynchronous calls on `stream`, device-detected errors through a sync call).
 *
 * Per image: h = patch_conv(image) + position embedding (a 14 x 14, stride 14 convolution
 * 3 -> 1152 with bias; tokens in raster order of the 16 x 16 patch grid); n_layers pre-norm
 * layers h += o_proj(MHA(LN1(h))), h += fc2(GELU_tanh(fc1(LN2(h)))) with biased q/k/v/o/fc1/
 * fc2 linears and bidirectional attention over the image's 256 tokens (16 heads x 72, scale
 * 1/sqrt(72), no mask, no rotary embedding); then embeddings = sqrt(2048) *
 * (post_LN(h) W_proj^T + b_proj).  LayerNorm: (x - mean) / sqrt(var + ln_eps) * w + b,
 * biased variance.  The pages name the tower; patch 14, 16 heads and MLP 4304 are the public
 * SigLIP-So400m/14 shape, which has the pages' 27 layers, width 1152 and ~400M parameters.
 * ========================================================================================= */
typedef struct rtvla_vision_ctx rtvla_vision_ctx; /* opaque; owned by the library */

typedef struct {
  int n_layers;   /* 27 (1..64 accepted) */
  int width;      /* 1152 */
  int mlp_dim;    /* 4304 */
  int n_heads;    /* 16 (head_dim = width / n_heads = 72) */
  int patch;      /* 14 */
  int image;      /* 224: (image / patch)^2 = 256 tokens per image, 3 channels */
  int out_width;  /* 2048: the prefix pass's width */
  int max_images; /* most images one rtvla_encode_images call encodes (1..64) */
  float ln_eps;   /* 1e-6 */
} rtvla_vision_config;

/* Device pointers to bf16 tensors, read only during rtvla_vision_create (the library keeps its
 * own repacked copies).  Per-layer fields are host arrays of n_layers device pointers. */
typedef struct {
  const void *patch_w;          /* [width][3][patch][patch] patch convolution */
  const void *patch_b;          /* [width] */
  const void *pos;              /* [256][width] position embedding */
  const void *const *ln1_w;     /* [L] -> [width]  LayerNorm before attention: gain */
  const void *const *ln1_b;     /* [L] -> [width]  offset */
  const void *const *wq;        /* [L] -> [width][width] */
  const void *const *bq;        /* [L] -> [width] */
  const void *const *wk;
  const void *const *bk;
  const void *const *wv;
  const void *const *bv;
  const void *const *wo;        /* [L] -> [width][width] attention output projection */
  const void *const *bo;
  const void *const *ln2_w;     /* [L] -> [width]  LayerNorm before the MLP */
  const void *const *ln2_b;
  const void *const *fc1_w;     /* [L] -> [mlp_dim][width] */
  const void *const *fc1_b;     /* [L] -> [mlp_dim] */
  const void *const *fc2_w;     /* [L] -> [width][mlp_dim] */
  const void *const *fc2_b;     /* [L] -> [width] */
  const void *post_w;           /* [width] post_layernorm gain */
  const void *post_b;           /* [width] */
  const void *proj_w;           /* [out_width][width] multi_modal_projector */
  const void *proj_b;           /* [out_width] */
} rtvla_vision_weights;

/* Creates an image-encoder context: repacks the weights (fc1 / fc2 zero-padded to 4352 MLP
 * features, the patch operand to 640 values), builds the fp32 table patch bias + position
 * embedding, and allocates every buffer for max_images images.  Synchronous.  Errors:
 * INVALID_ARG, UNSUPPORTED (a shape other than the one above), OOM, CUDA.  Reads
 * RTVLA_WAIT_TIMEOUT_US, RTVLA_CHECKED and RTVLA_DEVICE_MEMORY_CAP as rtvla_create does. */
rtvla_status rtvla_vision_create(const rtvla_vision_weights *w, const rtvla_vision_config *cfg,
                                 rtvla_vision_ctx **out);

/*
 * Encodes batch x views images and writes their embeddings into the prefix buffer of
 * rtvla_prefill.  images: device f32 [batch][views][3][224][224], pixels after resize and
 * [-1, 1] normalisation, 4-byte aligned.  prefix_embeds: device bf16
 * [batch][prefix_len][out_width], 16-byte aligned: view v of sample b fills rows
 * v * 256 .. v * 256 + 255 of sample b; no other row is written (the caller puts the prompt
 * embeddings after the image rows).  Runs as one CUDA-graph replay per call (captured on the
 * first call with this image count).  Errors: INVALID_ARG (null or misaligned pointer, batch
 * or views < 1), SHAPE (batch * views > max_images, or views * 256 > prefix_len);
 * device-detected DEVICE_TIMEOUT through rtvla_vision_sync_status.
 */
rtvla_status rtvla_encode_images(rtvla_vision_ctx *ctx, const float *images, int batch, int views,
                                 void *prefix_embeds, int prefix_len, void *stream);

/* Test hook: encodes n_images images of [n][3][224][224] (as one sample of n views) and
 * writes the residual stream after the embedding and after each layer to h_layers: device f32
 * [n_layers + 1][n_images * 256][width]; then the embeddings to prefix_embeds as
 * rtvla_encode_images would (prefix_len = n_images * 256).  Launches the kernels directly
 * (no graph).  Errors: as rtvla_encode_images. */
rtvla_status rtvla_vision_debug_trace(rtvla_vision_ctx *ctx, const float *images, int n_images,
                                      float *h_layers, void *prefix_embeds, void *stream);

/* As rtvla_sync_status, for an image-encoder context (guard bands checked in checked mode). */
rtvla_status rtvla_vision_sync_status(rtvla_vision_ctx *ctx, void *stream);

/* Kernels of this library one rtvla_encode_images call of n_images images launches (after
 * such a call has been made once), else -1. */
int rtvla_vision_kernels_per_call(rtvla_vision_ctx *ctx, int n_images);

/* Frees everything the context owns (waits for the device first).  NULL is a no-op. */
void rtvla_vision_destroy(rtvla_vision_ctx *ctx);

#ifdef __cplusplus
}
#endif

#endif /* RTVLA_H */
