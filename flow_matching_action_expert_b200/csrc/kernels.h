// Host-side launchers of the rtvla kernels (internal to librtvla.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace rtvla {

// ---------------------------------------------------------------------------------------
// tcgen05 skinny GEMM
struct GemmParams {
  int M, N, K;
  int w_row0;          // first row of this weight in the stacked tensor map
  int kb_per_split;    // 64-wide K blocks per CTA
  float *out;
  int ldo;
  const float *col_scale;  // per-output-column factor (AdaRMS gate) or null
  int atomic;              // 1: fp32 reduction into out; 0: plain store
  DevCtl *ctl;
  int m_tiles, n_tiles, splits;  // the launch's tiles (a CTA loops over tile c, c + grid, ...)
  // gated-GELU epilogue (glu = 1): the weight is [gate rows ; up rows] (N = 2F); tile n holds
  // gate rows n*64 .. n*64+63 and the matching up rows, and the epilogue writes
  // bf16 GELU_tanh(r*g + b_g) * (r*u + b_u) for features n*64 .. n*64+63 (r per token row,
  // b from glu_bias [2F]; either may be null) through a bf16 map of the [M][F] output
  int glu;
  const float *glu_r;
  const float *glu_bias;
};

struct GemmPlan {
  int tn, m_tiles, n_tiles, splits, kb_per_split;
};

// One activation tensor map per token tile (box heights 64, 128, 256): the box must match
// the tile the plan picks for the call's row count.
struct XMaps {
  CUtensorMap m[3];
};
int gemm_tile_index(int tn);
GemmPlan gemm_plan(int M, int N, int K, int sm_count);
cudaError_t gemm_init_attributes();
// The 2-CTA form (gemm_tc2.cu): 256 weight rows x 256 tokens per SM pair.  Init records how
// many 2-CTA clusters fit at once (0 disables the form); with RTVLA_PAIR_GEMM=1 set at init,
// gemm_launch picks it for token tiles of 256 when N is a multiple of 256.
cudaError_t gemm2_init_attributes(int sm_count);
int gemm2_clusters();
cudaError_t gemm2_launch(const CUtensorMap &tmW, const CUtensorMap &tmX128, const CUtensorMap &tmO,
                         const GemmParams &p, cudaStream_t st);

// Gated-GELU form of gemm_launch: m[t][f] = GELU_tanh(r[t] g + b_g[f]) * (r[t] u + b_u[f]) with
// g, u = X W^T over the gate rows w_row0 + f and the up rows w_row0 + F + f of tmW64 (a map
// with 64-row boxes); written as bf16 through tmM (64 x 64 boxes, 128-byte swizzle).  Needs
// the whole K in one tile: returns false (nothing launched) when the plan would split K.
bool gemm_glu_applies(int M, int F, int K, int sm_count);
cudaError_t gemm_launch_glu(const CUtensorMap &tmW64, int w_row0, const XMaps &xm, int M, int F, int K,
                            const CUtensorMap &tmM, const float *r, const float *bias, DevCtl *ctl, int sm_count,
                            cudaStream_t st);

// out[m][n] (+)= col_scale[n] * sum_k X[m][k] W[w_row0 + n][k].  `accumulate` adds into the
// existing contents of out; otherwise out must be zero when the plan splits K.
// tmO: fp32 map of `out` ([rows][ldo], 128-column x 64-row boxes, no swizzle)
cudaError_t gemm_launch(const CUtensorMap &tmW, int w_row0, const XMaps &xm, int M, int N, int K, float *out,
                        const CUtensorMap &tmO, int ldo, const float *col_scale, bool accumulate, DevCtl *ctl,
                        int sm_count, cudaStream_t st);

// ---------------------------------------------------------------------------------------
// attention (8 query heads share one KV head, head_dim 256)
struct AttnParams {
  const bf16 *q;            // [rows][q_ld], head h at column h*256; row = b*nq + i
  int q_ld;
  const CallArgs *ca;       // prefix K/V, valid lengths and cache stride of this call
  int layer;
  const bf16 *ksuf;         // suffix K/V [batch][n_suf][256] (may be null when n_suf = 0)
  const bf16 *vsuf;
  int n_suf;
  int nq;                   // queries per sample
  int keys_per_split;       // multiple of 64
  int n_splits;
  float *opart;             // [B][splits][nq][8][256] unnormalised partial outputs
  float *mlpart;            // [B][splits][nq][8][2]   (running max in log2 units, sum)
  bf16 *out;                // [rows][2048]
  float scale_log2;         // log2(e) / sqrt(head_dim)
  DevCtl *ctl;
};

cudaError_t attn_init_attributes();
int attn_splits(int batch, int nq, int max_keys, int sm_count, int *keys_per_split);
// Keys the split plan must cover: prefix and suffix are chunked separately (64 keys each).
int attn_keys(int prefix_cap, int n_suf);
cudaError_t attn_launch(const AttnParams &p, int batch, cudaStream_t st);
cudaError_t attn_tc_init_attributes();
cudaError_t attn_tc_launch(const AttnParams &p, int batch, cudaStream_t st);

// ---------------------------------------------------------------------------------------
// element-wise / row kernels
cudaError_t launch_init_x(const CallArgs *ca, float *x, int n, int Ct, int first, cudaStream_t st);
cudaError_t launch_pi0_in(const float *x, const float *w_fold, const float *c_k, const bf16 *w_st, const float *b_st,
                          const float *b_ato, const CallArgs *ca, float *h, bf16 *op, int M, int Ct, cudaStream_t st);
cudaError_t launch_action_in(const float *x, const bf16 *w_in, const float *b_in, float *h, int M,
                             cudaStream_t st);
cudaError_t launch_adanorm(const float *h, const float *s1p, bf16 *op, float *r, int M, float eps,
                           cudaStream_t st);
cudaError_t launch_qkv_post(float *acc, const float *r, const float *bias, const CallArgs *ca, int C,
                            const float *rope_cos, const float *rope_sin, int rope_rows, bf16 *q, bf16 *ks,
                            bf16 *vs, int M, DevCtl *ctl, cudaStream_t st);
cudaError_t launch_gelu_mul(float *acc, const float *r, const float *bias, bf16 *out, int M, int F,
                            cudaStream_t st);
cudaError_t launch_final(const float *h, const float *s1p, const float *shift, const float *w_out,
                         const float *b_out, float *x, int M, int final_norm, float eps, const CallArgs *ca,
                         int write_actions, int Ct, int first, cudaStream_t st);
// prefix pass
cudaError_t launch_pf_mask(const CallArgs *ca, int B, int P, DevCtl *ctl, cudaStream_t st);
cudaError_t launch_pf_embed(const CallArgs *ca, float *x, int M, int Dp, cudaStream_t st);
cudaError_t launch_rmsnorm(const float *x, bf16 *op, int M, int Dp, float eps, cudaStream_t st);
cudaError_t launch_pf_qkv_post(float *acc, const CallArgs *ca, int layer, int P, const float *rope_cos,
                               const float *rope_sin, int rope_rows, bf16 *q, int M, DevCtl *ctl, cudaStream_t st);

// ---------------------------------------------------------------------------------------
// create-time precompute (fp64)
cudaError_t launch_rows_dot_f64(const bf16 *W, int R, int Kd, const double *vecs, int S, const bf16 *bias,
                                double *out, cudaStream_t st);
cudaError_t launch_fold_cols(const bf16 *W, int R, int Kd, const bf16 *gamma, bf16 *out, cudaStream_t st);
cudaError_t launch_scale_to_f32(const bf16 *w, int n, double s, float *out, cudaStream_t st);

// ---------------------------------------------------------------------------------------
// image front-end (vision.cu): SigLIP-shaped tower of width 1152, 16 heads x 72, 256 tokens per
// 224 x 224 image (14 x 14 patches), projector to 2048
constexpr int VIS_WIDTH = 1152;
constexpr int VIS_TOKENS = 256;
constexpr int VIS_PATCH_K = 640;   // the patch operand's 3 x 14 x 14 = 588 values, zero-padded
constexpr int VIS_MLP_PAD = 4352;  // the MLP width 4304, zero-padded to whole 128-row tiles
constexpr int VIS_OUT = 2048;

// Per-call pointers of the captured encode graph (written to device memory before each replay).
struct VisArgs {
  const float *images;  // [n][3][224][224]
  bf16 *out;            // prefix embeddings [batch][ld][2048]
  int views;            // image i -> sample i / views, rows (i % views) * 256 ..
  int ld;               // prefix rows per sample
};

cudaError_t vis_init_attributes();
cudaError_t launch_vis_embed(const VisArgs *va, bf16 *cols, float *h, const float *table, int n_img,
                             cudaStream_t st);
cudaError_t launch_vis_ln(float *x, const float *add, const float *gain, const float *offset, bf16 *y, float *acc,
                          const float *acc_init, int acc_cols, int M, float eps, cudaStream_t st);
cudaError_t launch_vis_attn(const float *qkv, bf16 *out, int n_img, cudaStream_t st);
cudaError_t launch_vis_gelu(const float *acc, bf16 *out, int M, int cols, cudaStream_t st);
cudaError_t launch_vis_out(const VisArgs *va, const float *acc, int n_img, cudaStream_t st);

// ---------------------------------------------------------------------------------------
// checked mode: guard bands of GUARD_BYTES filled with GUARD_FILL before and after every
// library buffer; the checker flags (DEVERR_GUARD) and refills every band that changed
constexpr int GUARD_BYTES = 4096;
constexpr unsigned char GUARD_FILL = 0xA5;
struct GuardRegion {
  unsigned char *base;       // front band at [base, base + GUARD_BYTES)
  unsigned long long bytes;  // buffer bytes (a multiple of 256); back band right after them
};
cudaError_t launch_check_guards(const GuardRegion *regions, int n, DevCtl *ctl, cudaStream_t st);

}  // namespace rtvla
