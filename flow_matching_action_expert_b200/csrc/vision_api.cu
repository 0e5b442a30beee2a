// C ABI of the image front-end (rtvla_vision_*): the SigLIP-shaped vision tower and the
// multi_modal_projector of the Realtime-VLA tech blog ("pi0.5 inference flow": model
// structure, encoder step 1, class hierarchy).
//
// rtvla_vision_create repacks the weights into three stacked bf16 tensors, one per GEMM K
// width (1152: [q; k; v], o, fc1 of every layer, then the projector; 4352: fc2; 640: the patch
// convolution), keeps every bias, LayerNorm affine and the patch-bias + position table in
// fp32, and allocates the activations once for max_images images (the blog's "Static
// buffers").  rtvla_encode_images replays one CUDA graph per image count (the blog's "CUDA
// Graph": inputs written to a device argument block, then one replay).
//
// Per layer: k_vis_ln (LN1; h += b_o; acc := b_qkv) -> GEMM QKV into acc -> k_vis_attn ->
// GEMM O into h -> k_vis_ln (LN2; h += b_fc2; acc := b_fc1) -> GEMM fc1 into acc ->
// k_vis_gelu -> GEMM fc2 into h.  Every GEMM reduces into a buffer that already holds its
// bias (or the residual stream plus the bias), so no GEMM needs a bias epilogue.
#include <cudaTypedefs.h>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <map>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "rtvla.h"

using namespace rtvla;

namespace {
constexpr int VW = VIS_WIDTH;          // 1152
constexpr int VF = 4304;               // MLP width
constexpr int VFP = VIS_MLP_PAD;       // 4352
constexpr int VQKV = 3 * VW;           // 3456
constexpr int VT = VIS_TOKENS;         // 256
constexpr int VKP = VIS_PATCH_K;       // 640
constexpr int VKR = 588;               // 3 x 14 x 14
constexpr int VOUT = VIS_OUT;          // 2048
constexpr int VROWS = VQKV + VW + VFP; // rows of one layer in the K = 1152 stack
}  // namespace

struct rtvla_vision_ctx {
  rtvla_vision_config cfg;
  int device = 0, sm_count = 148, L = 0, NI = 0;
  std::vector<void *> allocs;
  size_t mem_cap = 0, mem_used = 0;
  bool checked = false;
  std::vector<GuardRegion> guards;
  GuardRegion *d_guards = nullptr;
  // weights (library-owned)
  bf16 *w_a = nullptr, *w_b = nullptr, *w_p = nullptr;
  float *b_qkv = nullptr, *b_o = nullptr, *b_fc1 = nullptr, *b_fc2 = nullptr;
  float *ln1_g = nullptr, *ln1_b = nullptr, *ln2_g = nullptr, *ln2_b = nullptr;
  float *post_g = nullptr, *post_b = nullptr, *b_proj = nullptr, *table = nullptr;
  // activations (NI * 256 rows)
  bf16 *cols = nullptr, *xn = nullptr, *ao = nullptr, *mb = nullptr;
  float *h = nullptr, *acc = nullptr;
  // control
  DevCtl *ctl = nullptr;
  VisArgs *args = nullptr;
  CUtensorMap tm_wa, tm_wb, tm_wp, tmo_h, tmo_qkv, tmo_fc1, tmo_proj;
  XMaps xm_cols, xm_xn, xm_ao, xm_mb;
  std::map<int, std::pair<cudaGraphExec_t, int>> graphs;
  cudaStream_t cap_stream = nullptr;
};

namespace {

PFN_cuTensorMapEncodeTiled_v12000 v_encode = nullptr;

bool v_get_encoder() {
  if (v_encode) return true;
  cudaDriverEntryPointQueryResult q;
  void *fn = nullptr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return false;
  v_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

// bf16 [rows][cols], 64-column x box_rows boxes, 128-byte swizzle (GEMM operands)
bool v_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return v_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 [rows][cols], 128-column x 64-row boxes, no swizzle (GEMM bulk-reduce targets)
bool v_map_out(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {128, 64};
  cuuint32_t es[2] = {1, 1};
  return v_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool v_xmaps(XMaps *x, const void *base, uint64_t rows, uint64_t cols) {
  return v_map(&x->m[0], base, rows, cols, 64) && v_map(&x->m[1], base, rows, cols, 128) &&
         v_map(&x->m[2], base, rows, cols, 256);
}

// Allocation with the context's memory cap and, in checked mode, guard bands (as the denoise
// context's buffers).
template <typename T>
T *v_alloc(rtvla_vision_ctx *c, size_t n) {
  void *p = nullptr;
  if (n == 0) n = 1;
  const size_t bytes = (n * sizeof(T) + 255) & ~size_t(255);
  const size_t total = c->checked ? bytes + 2 * (size_t)GUARD_BYTES : bytes;
  if (c->mem_cap && c->mem_used + total > c->mem_cap) return nullptr;
  if (cudaMalloc(&p, total) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  c->allocs.push_back(p);
  c->mem_used += total;
  if (!c->checked) return static_cast<T *>(p);
  unsigned char *b = static_cast<unsigned char *>(p);
  if (cudaMemset(b, GUARD_FILL, GUARD_BYTES) != cudaSuccess ||
      cudaMemset(b + GUARD_BYTES + bytes, GUARD_FILL, GUARD_BYTES) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  c->guards.push_back(GuardRegion{b, (unsigned long long)bytes});
  return reinterpret_cast<T *>(b + GUARD_BYTES);
}

void v_free(rtvla_vision_ctx *c) {
  for (auto &g : c->graphs)
    if (g.second.first) cudaGraphExecDestroy(g.second.first);
  for (void *p : c->allocs) cudaFree(p);
  if (c->d_guards) cudaFree(c->d_guards);
  if (c->cap_stream) cudaStreamDestroy(c->cap_stream);
  delete c;
}

bool v_shape_ok(const rtvla_vision_config *g) {
  return g->width == VW && g->mlp_dim == VF && g->n_heads == 16 && g->patch == 14 && g->image == 224 &&
         g->out_width == VOUT;
}

bool v_weights_present(const rtvla_vision_weights *w, int L) {
  if (!w->patch_w || !w->patch_b || !w->pos || !w->post_w || !w->post_b || !w->proj_w || !w->proj_b) return false;
  const void *const *per[] = {w->ln1_w, w->ln1_b, w->wq, w->bq, w->wk, w->bk, w->wv, w->bv,
                              w->wo,    w->bo,    w->ln2_w, w->ln2_b, w->fc1_w, w->fc1_b, w->fc2_w, w->fc2_b};
  for (const void *const *a : per) {
    if (!a) return false;
    for (int l = 0; l < L; ++l)
      if (!a[l]) return false;
  }
  return true;
}

cudaError_t to_f32(const void *src, int n, float *dst) {
  return launch_scale_to_f32(static_cast<const bf16 *>(src), n, 1.0, dst, 0);
}

float bf16_bits_to_f32(uint16_t b) {
  const uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

rtvla_status v_create_impl(rtvla_vision_ctx *c, const rtvla_vision_weights *w) {
  const int L = c->L;
  const size_t T = (size_t)c->NI * VT;
  if (cudaGetDevice(&c->device) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess)
    return RTVLA_ERR_CUDA;
  if (!v_get_encoder()) return RTVLA_ERR_CUDA;
  if (gemm_init_attributes() != cudaSuccess || vis_init_attributes() != cudaSuccess) return RTVLA_ERR_CUDA;
  if (cudaStreamCreateWithFlags(&c->cap_stream, cudaStreamNonBlocking) != cudaSuccess) return RTVLA_ERR_CUDA;

  // ---- weights
  const size_t rows_a = (size_t)L * VROWS + VOUT;
  c->w_a = v_alloc<bf16>(c, rows_a * VW);
  c->w_b = v_alloc<bf16>(c, (size_t)L * VW * VFP);
  c->w_p = v_alloc<bf16>(c, (size_t)VW * VKP);
  c->b_qkv = v_alloc<float>(c, (size_t)L * VQKV);
  c->b_o = v_alloc<float>(c, (size_t)L * VW);
  c->b_fc1 = v_alloc<float>(c, (size_t)L * VFP);
  c->b_fc2 = v_alloc<float>(c, (size_t)L * VW);
  c->ln1_g = v_alloc<float>(c, (size_t)L * VW);
  c->ln1_b = v_alloc<float>(c, (size_t)L * VW);
  c->ln2_g = v_alloc<float>(c, (size_t)L * VW);
  c->ln2_b = v_alloc<float>(c, (size_t)L * VW);
  c->post_g = v_alloc<float>(c, VW);
  c->post_b = v_alloc<float>(c, VW);
  c->b_proj = v_alloc<float>(c, VOUT);
  c->table = v_alloc<float>(c, (size_t)VT * VW);
  if (!c->w_a || !c->w_b || !c->w_p || !c->b_qkv || !c->b_o || !c->b_fc1 || !c->b_fc2 || !c->ln1_g || !c->ln1_b ||
      !c->ln2_g || !c->ln2_b || !c->post_g || !c->post_b || !c->b_proj || !c->table)
    return RTVLA_ERR_OOM;
  // zero padding: fc1 rows 4304.., fc2 columns 4304.., patch columns 588.., the fc1 bias tail
  if (cudaMemset(c->w_a, 0, rows_a * VW * 2) != cudaSuccess ||
      cudaMemset(c->w_b, 0, (size_t)L * VW * VFP * 2) != cudaSuccess ||
      cudaMemset(c->w_p, 0, (size_t)VW * VKP * 2) != cudaSuccess ||
      cudaMemset(c->b_fc1, 0, (size_t)L * VFP * 4) != cudaSuccess)
    return RTVLA_ERR_CUDA;
  const cudaMemcpyKind dd = cudaMemcpyDeviceToDevice;
  const size_t sq = (size_t)VW * VW * 2;
  for (int l = 0; l < L; ++l) {
    bf16 *a = c->w_a + (size_t)l * VROWS * VW;
    if (cudaMemcpy(a, w->wq[l], sq, dd) != cudaSuccess || cudaMemcpy(a + (size_t)VW * VW, w->wk[l], sq, dd) != cudaSuccess ||
        cudaMemcpy(a + (size_t)2 * VW * VW, w->wv[l], sq, dd) != cudaSuccess ||
        cudaMemcpy(a + (size_t)VQKV * VW, w->wo[l], sq, dd) != cudaSuccess ||
        cudaMemcpy(a + (size_t)(VQKV + VW) * VW, w->fc1_w[l], (size_t)VF * VW * 2, dd) != cudaSuccess ||
        cudaMemcpy2D(c->w_b + (size_t)l * VW * VFP, (size_t)VFP * 2, w->fc2_w[l], (size_t)VF * 2, (size_t)VF * 2, VW,
                     dd) != cudaSuccess)
      return RTVLA_ERR_CUDA;
    if (to_f32(w->bq[l], VW, c->b_qkv + (size_t)l * VQKV) != cudaSuccess ||
        to_f32(w->bk[l], VW, c->b_qkv + (size_t)l * VQKV + VW) != cudaSuccess ||
        to_f32(w->bv[l], VW, c->b_qkv + (size_t)l * VQKV + 2 * VW) != cudaSuccess ||
        to_f32(w->bo[l], VW, c->b_o + (size_t)l * VW) != cudaSuccess ||
        to_f32(w->fc1_b[l], VF, c->b_fc1 + (size_t)l * VFP) != cudaSuccess ||
        to_f32(w->fc2_b[l], VW, c->b_fc2 + (size_t)l * VW) != cudaSuccess ||
        to_f32(w->ln1_w[l], VW, c->ln1_g + (size_t)l * VW) != cudaSuccess ||
        to_f32(w->ln1_b[l], VW, c->ln1_b + (size_t)l * VW) != cudaSuccess ||
        to_f32(w->ln2_w[l], VW, c->ln2_g + (size_t)l * VW) != cudaSuccess ||
        to_f32(w->ln2_b[l], VW, c->ln2_b + (size_t)l * VW) != cudaSuccess)
      return RTVLA_ERR_CUDA;
  }
  if (cudaMemcpy(c->w_a + (size_t)L * VROWS * VW, w->proj_w, (size_t)VOUT * VW * 2, dd) != cudaSuccess ||
      cudaMemcpy2D(c->w_p, (size_t)VKP * 2, w->patch_w, (size_t)VKR * 2, (size_t)VKR * 2, VW, dd) != cudaSuccess ||
      to_f32(w->post_w, VW, c->post_g) != cudaSuccess || to_f32(w->post_b, VW, c->post_b) != cudaSuccess ||
      to_f32(w->proj_b, VOUT, c->b_proj) != cudaSuccess)
    return RTVLA_ERR_CUDA;
  // residual-stream start: patch bias + position embedding, fp32 [256][1152]
  {
    std::vector<uint16_t> pos((size_t)VT * VW), pb(VW);
    if (cudaMemcpy(pos.data(), w->pos, pos.size() * 2, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(pb.data(), w->patch_b, pb.size() * 2, cudaMemcpyDeviceToHost) != cudaSuccess)
      return RTVLA_ERR_CUDA;
    std::vector<float> tab(pos.size());
    for (size_t i = 0; i < tab.size(); ++i) tab[i] = bf16_bits_to_f32(pos[i]) + bf16_bits_to_f32(pb[i % VW]);
    if (cudaMemcpy(c->table, tab.data(), tab.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess) return RTVLA_ERR_CUDA;
  }

  // ---- activations and control
  c->cols = v_alloc<bf16>(c, T * VKP);
  c->h = v_alloc<float>(c, T * VW);
  c->xn = v_alloc<bf16>(c, T * VW);
  c->ao = v_alloc<bf16>(c, T * VW);
  c->acc = v_alloc<float>(c, T * VFP);
  c->mb = v_alloc<bf16>(c, T * VFP);
  c->ctl = v_alloc<DevCtl>(c, 1);
  c->args = v_alloc<VisArgs>(c, 1);
  if (!c->cols || !c->h || !c->xn || !c->ao || !c->acc || !c->mb || !c->ctl || !c->args) return RTVLA_ERR_OOM;
  DevCtl hc;
  std::memset(&hc, 0, sizeof(hc));
  hc.timeout_ns = 2000000000ull;
  if (const char *env = std::getenv("RTVLA_WAIT_TIMEOUT_US")) {
    const long long us = std::atoll(env);
    if (us > 0) hc.timeout_ns = (unsigned long long)us * 1000ull;
  }
  if (cudaMemcpy(c->ctl, &hc, sizeof(hc), cudaMemcpyHostToDevice) != cudaSuccess) return RTVLA_ERR_CUDA;

  // ---- tensor maps (weights: 128-row boxes; operands: one map per token-tile height)
  const bool ok = v_map(&c->tm_wa, c->w_a, rows_a, VW, 128) && v_map(&c->tm_wb, c->w_b, (uint64_t)L * VW, VFP, 128) &&
                  v_map(&c->tm_wp, c->w_p, VW, VKP, 128) && v_xmaps(&c->xm_cols, c->cols, T, VKP) &&
                  v_xmaps(&c->xm_xn, c->xn, T, VW) && v_xmaps(&c->xm_ao, c->ao, T, VW) &&
                  v_xmaps(&c->xm_mb, c->mb, T, VFP) && v_map_out(&c->tmo_h, c->h, T, VW) &&
                  v_map_out(&c->tmo_qkv, c->acc, T, VQKV) && v_map_out(&c->tmo_fc1, c->acc, T, VFP) &&
                  v_map_out(&c->tmo_proj, c->acc, T, VOUT);
  if (!ok) return RTVLA_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return RTVLA_ERR_CUDA;
  return RTVLA_OK;
}

#define VCK(x)                        \
  do {                                \
    cudaError_t e_ = (x);             \
    if (e_ != cudaSuccess) return e_; \
    ++n;                              \
  } while (0)

// The encode pass for n_img images (kernels read the call's pointers from c->args).  trace:
// when given, h after the embedding and after each layer is copied there.
cudaError_t v_enqueue(rtvla_vision_ctx *c, int n_img, cudaStream_t st, float *trace, int *kernels) {
  int n = 0;
  const int L = c->L, M = n_img * VT, sm = c->sm_count;
  const float eps = c->cfg.ln_eps;
  const size_t hb = (size_t)M * VW * 4;
  VCK(launch_vis_embed(c->args, c->cols, c->h, c->table, n_img, st));
  VCK(gemm_launch(c->tm_wp, 0, c->xm_cols, M, VW, VKP, c->h, c->tmo_h, VW, nullptr, true, c->ctl, sm, st));
  if (trace) {
    const cudaError_t e = cudaMemcpyAsync(trace, c->h, hb, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
  }
  for (int l = 0; l < L; ++l) {
    const int r0 = l * VROWS;
    VCK(launch_vis_ln(c->h, c->b_o + (size_t)l * VW, c->ln1_g + (size_t)l * VW, c->ln1_b + (size_t)l * VW, c->xn,
                      c->acc, c->b_qkv + (size_t)l * VQKV, VQKV, M, eps, st));
    VCK(gemm_launch(c->tm_wa, r0, c->xm_xn, M, VQKV, VW, c->acc, c->tmo_qkv, VQKV, nullptr, true, c->ctl, sm, st));
    VCK(launch_vis_attn(c->acc, c->ao, n_img, st));
    VCK(gemm_launch(c->tm_wa, r0 + VQKV, c->xm_ao, M, VW, VW, c->h, c->tmo_h, VW, nullptr, true, c->ctl, sm, st));
    VCK(launch_vis_ln(c->h, c->b_fc2 + (size_t)l * VW, c->ln2_g + (size_t)l * VW, c->ln2_b + (size_t)l * VW, c->xn,
                      c->acc, c->b_fc1 + (size_t)l * VFP, VFP, M, eps, st));
    VCK(gemm_launch(c->tm_wa, r0 + VQKV + VW, c->xm_xn, M, VFP, VW, c->acc, c->tmo_fc1, VFP, nullptr, true, c->ctl,
                    sm, st));
    VCK(launch_vis_gelu(c->acc, c->mb, M, VFP, st));
    VCK(gemm_launch(c->tm_wb, l * VW, c->xm_mb, M, VW, VFP, c->h, c->tmo_h, VW, nullptr, true, c->ctl, sm, st));
    if (trace) {
      const cudaError_t e = cudaMemcpyAsync(trace + (size_t)(l + 1) * M * VW, c->h, hb, cudaMemcpyDeviceToDevice, st);
      if (e != cudaSuccess) return e;
    }
  }
  VCK(launch_vis_ln(c->h, nullptr, c->post_g, c->post_b, c->xn, c->acc, c->b_proj, VOUT, M, eps, st));
  VCK(gemm_launch(c->tm_wa, L * VROWS, c->xm_xn, M, VOUT, VW, c->acc, c->tmo_proj, VOUT, nullptr, true, c->ctl, sm, st));
  VCK(launch_vis_out(c->args, c->acc, n_img, st));
  if (kernels) *kernels = n;
  return cudaSuccess;
}

rtvla_status v_check_call(rtvla_vision_ctx *c, const float *images, int n_img, int views, const void *out,
                          int prefix_len) {
  if (!c || !images || !out || n_img < 1 || views < 1) return RTVLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(images) & 3) != 0 || (reinterpret_cast<uintptr_t>(out) & 15) != 0)
    return RTVLA_ERR_INVALID_ARG;
  if (n_img > c->NI || (long long)views * VT > prefix_len) return RTVLA_ERR_SHAPE;
  return RTVLA_OK;
}

rtvla_status v_write_args(rtvla_vision_ctx *c, const float *images, void *out, int views, int ld, cudaStream_t st) {
  VisArgs a;
  a.images = images;
  a.out = static_cast<bf16 *>(out);
  a.views = views;
  a.ld = ld;
  return cudaMemcpyAsync(c->args, &a, sizeof(a), cudaMemcpyHostToDevice, st) == cudaSuccess ? RTVLA_OK
                                                                                            : RTVLA_ERR_CUDA;
}

}  // namespace

// =======================================================================================
// C ABI

extern "C" {

rtvla_status rtvla_vision_create(const rtvla_vision_weights *w, const rtvla_vision_config *cfg, rtvla_vision_ctx **out) {
  if (!w || !cfg || !out) return RTVLA_ERR_INVALID_ARG;
  *out = nullptr;
  if (cfg->n_layers < 1 || cfg->n_layers > 64 || cfg->max_images < 1 || cfg->max_images > 64 || !(cfg->ln_eps >= 0.f))
    return RTVLA_ERR_INVALID_ARG;
  if (!v_shape_ok(cfg)) return RTVLA_ERR_UNSUPPORTED;
  if (!v_weights_present(w, cfg->n_layers)) return RTVLA_ERR_INVALID_ARG;
  rtvla_vision_ctx *c = new rtvla_vision_ctx();
  c->cfg = *cfg;
  c->L = cfg->n_layers;
  c->NI = cfg->max_images;
  if (const char *env = std::getenv("RTVLA_CHECKED")) c->checked = std::atoi(env) != 0;
  if (const char *env = std::getenv("RTVLA_DEVICE_MEMORY_CAP")) c->mem_cap = (size_t)std::strtoull(env, nullptr, 10);
  rtvla_status st = v_create_impl(c, w);
  if (st == RTVLA_OK && c->checked) {
    const size_t b = c->guards.size() * sizeof(GuardRegion);
    if (cudaMalloc(&c->d_guards, b) != cudaSuccess ||
        cudaMemcpy(c->d_guards, c->guards.data(), b, cudaMemcpyHostToDevice) != cudaSuccess)
      st = RTVLA_ERR_CUDA;
  }
  if (st != RTVLA_OK) {
    cudaGetLastError();
    v_free(c);
    return st;
  }
  *out = c;
  return RTVLA_OK;
}

rtvla_status rtvla_encode_images(rtvla_vision_ctx *c, const float *images, int batch, int views, void *prefix_embeds,
                                 int prefix_len, void *stream) {
  if (!c || batch < 1 || views < 1) return RTVLA_ERR_INVALID_ARG;
  const long long n = (long long)batch * views;
  if (n > c->NI) return RTVLA_ERR_SHAPE;
  rtvla_status s = v_check_call(c, images, (int)n, views, prefix_embeds, prefix_len);
  if (s != RTVLA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto it = c->graphs.find((int)n);
  if (it == c->graphs.end()) {
    cudaGraph_t g = nullptr;
    int k = 0;
    if (cudaStreamBeginCapture(c->cap_stream, cudaStreamCaptureModeThreadLocal) != cudaSuccess) return RTVLA_ERR_CUDA;
    const cudaError_t e = v_enqueue(c, (int)n, c->cap_stream, nullptr, &k);
    const cudaError_t e2 = cudaStreamEndCapture(c->cap_stream, &g);
    if (e != cudaSuccess || e2 != cudaSuccess || !g) {
      if (g) cudaGraphDestroy(g);
      cudaGetLastError();
      return RTVLA_ERR_CUDA;
    }
    cudaGraphExec_t ex = nullptr;
    const cudaError_t e3 = cudaGraphInstantiate(&ex, g, 0);
    cudaGraphDestroy(g);
    if (e3 != cudaSuccess) {
      cudaGetLastError();
      return RTVLA_ERR_CUDA;
    }
    it = c->graphs.emplace((int)n, std::make_pair(ex, k)).first;
  }
  s = v_write_args(c, images, prefix_embeds, views, prefix_len, st);
  if (s != RTVLA_OK) return s;
  return cudaGraphLaunch(it->second.first, st) == cudaSuccess ? RTVLA_OK : RTVLA_ERR_CUDA;
}

rtvla_status rtvla_vision_debug_trace(rtvla_vision_ctx *c, const float *images, int n_images, float *h_layers,
                                      void *prefix_embeds, void *stream) {
  if (!h_layers) return RTVLA_ERR_INVALID_ARG;
  rtvla_status s = v_check_call(c, images, n_images, n_images, prefix_embeds, n_images * VT);
  if (s != RTVLA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = v_write_args(c, images, prefix_embeds, n_images, n_images * VT, st);
  if (s != RTVLA_OK) return s;
  if (v_enqueue(c, n_images, st, h_layers, nullptr) != cudaSuccess) {
    cudaGetLastError();
    return RTVLA_ERR_CUDA;
  }
  return RTVLA_OK;
}

rtvla_status rtvla_vision_sync_status(rtvla_vision_ctx *c, void *stream) {
  if (!c) return RTVLA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (c->checked && launch_check_guards(c->d_guards, (int)c->guards.size(), c->ctl, st) != cudaSuccess) {
    cudaGetLastError();
    return RTVLA_ERR_CUDA;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return RTVLA_ERR_CUDA;
  }
  DevCtl h;
  if (cudaMemcpy(&h, c->ctl, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (h.err == 0) return RTVLA_OK;
  const int zero[2] = {0, 0};
  if (cudaMemcpy(c->ctl, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (h.err & DEVERR_TIMEOUT) return RTVLA_ERR_DEVICE_TIMEOUT;
  if (h.err & DEVERR_GUARD) return RTVLA_ERR_GUARD_OVERWRITE;
  return RTVLA_ERR_DEVICE_BOUNDS;
}

int rtvla_vision_kernels_per_call(rtvla_vision_ctx *c, int n_images) {
  if (!c) return -1;
  auto it = c->graphs.find(n_images);
  return it == c->graphs.end() ? -1 : it->second.second;
}

void rtvla_vision_destroy(rtvla_vision_ctx *c) {
  if (!c) return;
  cudaDeviceSynchronize();
  v_free(c);
}

}  // extern "C"
