// librtvla.so: the C ABI declared in include/rtvla.h.
//
// rtvla_create mirrors the Realtime-VLA "__init__" of the tech blog (section "Precompute
// (__init__)"): the time embedding + time MLP of the S fixed timesteps, every AdaRMS dense
// output for every (step, layer), Q/K/V concatenated into one weight, dt folded into
// action_out_proj, RoPE cos/sin tables, and every activation buffer allocated once
// (section "Static buffers").  rtvla_sample_actions mirrors "forward()" of section "CUDA
// Graph": the per-call pointers are copied into a device argument block and one captured
// graph (or one persistent kernel) runs the whole 10-step loop.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstddef>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "persistent.h"
#include "rtvla.h"

using namespace rtvla;

namespace {
struct GraphEntry {
  cudaGraphExec_t exec = nullptr;
  int kernels = 0;
};
constexpr int D = 1024, F = 4096, HD = 256, NQH = 8, A = 32, DP = 2048, FP = 16384;
}  // namespace

struct rtvla_ctx {
  rtvla_config cfg;
  int device = 0, sm_count = 148;
  // C: token rows per sample in the expert (the action chunk Ca, plus the state token for π0)
  int L = 0, S = 0, C = 0, Ca = 0, Bmax = 0, Pmax = 0;
  int variant = RTVLA_VARIANT_PI05, first = 0;  // first: rows before the action rows (π0: 1)
  int engine = RTVLA_ENGINE_AUTO;
  std::vector<void *> allocs;
  // folded / repacked expert weights (library-owned)
  bf16 *w_qkv = nullptr, *w_o = nullptr, *w_gu = nullptr, *w_d = nullptr, *w_in = nullptr;
  float *b_in = nullptr, *w_out = nullptr, *b_out = nullptr;
  // per-(step, layer) tables
  float *s1p_attn = nullptr, *gate_attn = nullptr, *s1p_ffn = nullptr, *gate_ffn = nullptr;
  float *bias_qkv = nullptr, *bias_gu = nullptr, *s1p_fin = nullptr, *shift_fin = nullptr;
  float *rope_cos = nullptr, *rope_sin = nullptr;
  int rope_rows = 0;
  // π0: folded action-time MLP (fp32 W_fold [D][A] and the pre-SiLU table c_k [S][D]), its
  // output linear (a GEMM weight), the state projection
  float *pi_wfold = nullptr, *pi_ctab = nullptr, *pi_bato = nullptr, *pi_bst = nullptr;
  bf16 *pi_wato = nullptr, *pi_wst = nullptr;
  CUtensorMap tm_wato;
  // prefix-pass weights
  bf16 *pw_qkv = nullptr, *pw_o = nullptr, *pw_gu = nullptr, *pw_d = nullptr;
  // denoise activations
  int Mmax = 0;
  float *x = nullptr, *h = nullptr, *r = nullptr, *acc_qkv = nullptr, *acc_gu = nullptr;
  float *opart = nullptr, *mlpart = nullptr;
  bf16 *op = nullptr, *q = nullptr, *ks = nullptr, *vs = nullptr, *o = nullptr, *mb = nullptr;
  // prefix-pass activations
  int Mpmax = 0;
  float *px = nullptr, *pacc = nullptr, *popart = nullptr, *pmlpart = nullptr;
  bf16 *pop = nullptr, *pq = nullptr, *po = nullptr, *pmb = nullptr;
  // persistent engine
  bool pers_ok = false;
  float *ss_attn = nullptr, *ss_ffn = nullptr, *pk_opart = nullptr, *pk_mlpart = nullptr;
  unsigned long long *pk_stamps = nullptr;
  int pk_max_phases = 0;
  // control
  DevCtl *ctl = nullptr;
  CallArgs *args_dn = nullptr, *args_pf = nullptr, *args_tr = nullptr;
  CUtensorMap tm_wqkv, tm_wo, tm_wgu, tm_wd, tm_pwqkv, tm_pwo, tm_pwgu, tm_pwd;
  CUtensorMap tm_wgu64, tm_pwgu64;  // the gate/up weights with 64-row boxes (gated-GELU GEMM)
  // fp32 GEMM outputs of the layered engine, 128-column x 64-row boxes (bulk store / reduce-add)
  CUtensorMap tmo_qkv, tmo_h, tmo_gu, tmo_pqkv, tmo_px, tmo_pgu;
  PersistMaps pmaps;                // tensor maps of the persistent engine
  CUtensorMap tm_q64;               // finalised Q, 64-row boxes
  const void *pk_cache_k = nullptr, *pk_cache_v = nullptr;  // prefix cache of the current call
  XMaps tm_op, tm_o, tm_mb, tm_pop, tm_po, tm_pmb;
  std::map<std::pair<int, int>, GraphEntry> graphs_dn, graphs_pf;
  std::map<int, int> kernels_per_call;
  cudaStream_t cap_stream = nullptr;
  // host-buffer staging (rtvla_sample_actions_host)
  bf16 *st_k = nullptr, *st_v = nullptr;
  int *st_vl = nullptr;
  float *st_noise = nullptr, *st_act = nullptr;
  size_t st_kv_elems = 0, st_io_elems = 0;
  int st_batch = 0;
  // checked mode (RTVLA_CHECKED=1 at create): guard bands around every library buffer
  bool checked = false;
  std::vector<GuardRegion> guards;
  GuardRegion *d_guards = nullptr;
  // device-memory cap of this context (RTVLA_DEVICE_MEMORY_CAP bytes at create; 0 = none)
  size_t mem_cap = 0, mem_used = 0;
};

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool get_encoder() {
  if (g_encode) return true;
  cudaDriverEntryPointQueryResult q;
  void *fn = nullptr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return false;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

// 2-D bf16 tensor [rows][cols] row-major, box = 64 columns x box_rows rows, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 [rows][cols] row-major; box = box_cols x 64 rows.  128-column boxes without swizzle
// are bulk-reduce targets; 32-column boxes with 128-byte swizzle are staging loads.
bool make_map_f32(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_cols, bool swz) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {box_cols, 64};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 [64][cols] row-major, seen as 3-D {32 columns, 64 rows, cols / 32 column blocks} with
// strides (row cols * 4 B, block 128 B): one box of `blocks` column blocks lands in shared
// memory as that many consecutive 8 KB tiles [64 rows][32 columns], each with 128-byte swizzle.
bool make_map_f32_blocks(CUtensorMap *m, const void *base, uint64_t cols, uint32_t blocks, uint64_t rows = 64) {
  cuuint64_t dims[3] = {32, rows, cols / 32};
  cuuint64_t strides[2] = {cols * 4, 128};
  cuuint32_t box[3] = {32, 64, blocks};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_xmaps(XMaps *x, const void *base, uint64_t rows, uint64_t cols) {
  return make_map(&x->m[0], base, rows, cols, 64) && make_map(&x->m[1], base, rows, cols, 128) &&
         make_map(&x->m[2], base, rows, cols, 256);
}

// Every buffer the context owns comes from here.  A context created with a device-memory
// cap refuses (nullptr, hence RTVLA_ERR_OOM) any allocation that would exceed it, exactly as
// a failed cudaMalloc would be handled.  In checked mode each buffer is placed between two
// guard bands of GUARD_BYTES filled with GUARD_FILL; rtvla_sync_status verifies them.
template <typename T>
T *dalloc(rtvla_ctx *c, size_t n) {
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

void free_all(rtvla_ctx *c) {
  for (auto &kv : c->graphs_dn)
    if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
  for (auto &kv : c->graphs_pf)
    if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
  for (void *p : c->allocs) cudaFree(p);
  if (c->d_guards) cudaFree(c->d_guards);
  if (c->st_k) cudaFree(c->st_k);
  if (c->st_v) cudaFree(c->st_v);
  if (c->st_vl) cudaFree(c->st_vl);
  if (c->st_noise) cudaFree(c->st_noise);
  if (c->st_act) cudaFree(c->st_act);
  if (c->cap_stream) cudaStreamDestroy(c->cap_stream);
  delete c;
}

std::vector<double> d2h_bf16(const void *p, size_t n) {
  std::vector<uint16_t> raw(n);
  std::vector<double> out(n);
  if (cudaMemcpy(raw.data(), p, n * 2, cudaMemcpyDeviceToHost) != cudaSuccess) return {};
  for (size_t i = 0; i < n; ++i) {
    uint32_t u = (uint32_t)raw[i] << 16;
    float f;
    std::memcpy(&f, &u, 4);
    out[i] = f;
  }
  return out;
}

double silu_d(double x) { return x / (1.0 + std::exp(-x)); }

bool valid_cfg(const rtvla_config *c) {
  if (c->n_layers < 1 || c->n_layers > 64 || c->n_steps < 1 || c->n_steps > 64) return false;
  if (c->chunk < 1 || c->chunk > 256 || c->max_batch < 1 || c->max_batch > 4096) return false;
  if (c->max_prefix < 1 || c->max_prefix > 65536) return false;
  if (c->engine < 0 || c->engine > 2) return false;
  if (c->variant != RTVLA_VARIANT_PI05 && c->variant != RTVLA_VARIANT_PI0) return false;
  if (c->variant == RTVLA_VARIANT_PI0 && c->chunk + 1 > 256) return false;
  if (!(c->rms_eps >= 0.f) || !(c->rope_theta > 0.f)) return false;
  return true;
}

bool supported_cfg(const rtvla_config *c) {
  if (c->width != D || c->mlp_dim != F || c->n_q_heads != NQH || c->n_kv_heads != 1 || c->head_dim != HD ||
      c->action_dim != A)
    return false;
  if (c->has_prefill && (c->pf_width != DP || c->pf_mlp_dim != FP)) return false;
  return true;
}

#define CKR(x)                                         \
  do {                                                 \
    cudaError_t e_ = (x);                              \
    if (e_ != cudaSuccess) return e_;                  \
  } while (0)
#define CKN(x)                                         \
  do {                                                 \
    cudaError_t e_ = (x);                              \
    if (e_ != cudaSuccess) return e_;                  \
    ++n;                                               \
  } while (0)

// ---------------------------------------------------------------------------------------
// layered engine: the denoise loop as a sequence of kernels (captured into one graph)
cudaError_t enqueue_denoise(rtvla_ctx *c, const CallArgs *dargs, int B, int cap, cudaStream_t st, float *trace,
                            int last_step, int *kernels) {
  int n = 0;
  const int L = c->L, S = c->S, C = c->C, M = B * C;
  const float eps = c->cfg.rms_eps;
  CKR(cudaMemsetAsync(c->acc_qkv, 0, (size_t)M * 2560 * 4, st));
  // the gate/up GEMM writes GELU(g) * u directly when its plan keeps K whole; otherwise it
  // accumulates into acc_gu (zeroed here; k_gelu_mul re-zeroes what it consumed)
  const bool glu = gemm_glu_applies(M, F, D, c->sm_count);
  if (!glu) CKR(cudaMemsetAsync(c->acc_gu, 0, (size_t)M * 2 * F * 4, st));
  CKN(launch_init_x(dargs, c->x, M * A, C, c->first, st));
  AttnParams ap;
  std::memset(&ap, 0, sizeof(ap));
  ap.q = c->q;
  ap.q_ld = NQH * HD;
  ap.ca = dargs;
  ap.ksuf = c->ks;
  ap.vsuf = c->vs;
  ap.n_suf = C;
  ap.nq = C;
  ap.n_splits = attn_splits(B, C, attn_keys(cap, C), c->sm_count, &ap.keys_per_split);
  ap.opart = c->opart;
  ap.mlpart = c->mlpart;
  ap.out = c->o;
  ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)HD));
  ap.ctl = c->ctl;
  const bool pi0 = c->variant == RTVLA_VARIANT_PI0;
  for (int k = 0; k <= last_step; ++k) {
    if (pi0) {
      // suffix rows: state projection; action tokens through the folded action-time MLP
      CKN(launch_pi0_in(c->x, c->pi_wfold, c->pi_ctab + (size_t)k * D, c->pi_wst, c->pi_bst, c->pi_bato, dargs, c->h,
                        c->op, M, C, st));
      CKN(gemm_launch(c->tm_wato, 0, c->tm_op, M, D, D, c->h, c->tmo_h, D, nullptr, true, c->ctl, c->sm_count, st));
    } else {
      CKN(launch_action_in(c->x, c->w_in, c->b_in, c->h, M, st));
    }
    if (trace && k == last_step)
      CKR(cudaMemcpyAsync(trace, c->h, (size_t)M * D * 4, cudaMemcpyDeviceToDevice, st));
    for (int l = 0; l < L; ++l) {
      const size_t kl = (size_t)k * L + l;
      CKN(launch_adanorm(c->h, c->s1p_attn + kl * D, c->op, c->r, M, eps, st));
      CKN(gemm_launch(c->tm_wqkv, l * 2560, c->tm_op, M, 2560, D, c->acc_qkv, c->tmo_qkv, 2560, nullptr, false, c->ctl,
                      c->sm_count, st));
      CKN(launch_qkv_post(c->acc_qkv, c->r, c->bias_qkv + kl * 2560, dargs, C, c->rope_cos, c->rope_sin,
                          c->rope_rows, c->q, c->ks, c->vs, M, c->ctl, st));
      ap.layer = l;
      CKN(attn_launch(ap, B, st));
      if (ap.n_splits > 1) ++n;
      CKN(gemm_launch(c->tm_wo, l * D, c->tm_o, M, D, NQH * HD, c->h, c->tmo_h, D, c->gate_attn + kl * D, true, c->ctl,
                      c->sm_count, st));
      CKN(launch_adanorm(c->h, c->s1p_ffn + kl * D, c->op, c->r, M, eps, st));
      if (glu) {
        CKN(gemm_launch_glu(c->tm_wgu64, l * 2 * F, c->tm_op, M, F, D, c->tm_mb.m[0], c->r, c->bias_gu + kl * 2 * F,
                            c->ctl, c->sm_count, st));
      } else {
        CKN(gemm_launch(c->tm_wgu, l * 2 * F, c->tm_op, M, 2 * F, D, c->acc_gu, c->tmo_gu, 2 * F, nullptr, false,
                        c->ctl, c->sm_count, st));
        CKN(launch_gelu_mul(c->acc_gu, c->r, c->bias_gu + kl * 2 * F, c->mb, M, F, st));
      }
      CKN(gemm_launch(c->tm_wd, l * D, c->tm_mb, M, D, F, c->h, c->tmo_h, D, c->gate_ffn + kl * D, true, c->ctl,
                      c->sm_count, st));
      if (trace && k == last_step)
        CKR(cudaMemcpyAsync(trace + (size_t)(l + 1) * M * D, c->h, (size_t)M * D * 4, cudaMemcpyDeviceToDevice,
                            st));
    }
    if (!trace)
      CKN(launch_final(c->h, c->s1p_fin + (size_t)k * D, c->shift_fin + (size_t)k * D, c->w_out, c->b_out, c->x, M,
                       c->cfg.final_norm, eps, dargs, k == S - 1 ? 1 : 0, C, c->first, st));
    else if (k < last_step)
      CKN(launch_final(c->h, c->s1p_fin + (size_t)k * D, c->shift_fin + (size_t)k * D, c->w_out, c->b_out, c->x, M,
                       c->cfg.final_norm, eps, dargs, 0, C, c->first, st));
  }
  *kernels = n;
  return cudaSuccess;
}

cudaError_t enqueue_prefill(rtvla_ctx *c, const CallArgs *dargs, int B, int P, cudaStream_t st, int *kernels) {
  int n = 0;
  const int L = c->L, M = B * P;
  const float eps = c->cfg.rms_eps;
  // the QKV accumulator (the first M x 2560 floats of pacc) must start at zero, and the
  // gate/up accumulator too unless the gate/up GEMM writes GELU(g) * u directly
  const bool glu = gemm_glu_applies(M, FP, DP, c->sm_count);
  CKR(cudaMemsetAsync(c->pacc, 0, (size_t)M * (glu ? 2560 : 2 * FP) * 4, st));
  CKN(launch_pf_mask(dargs, B, P, c->ctl, st));
  CKN(launch_pf_embed(dargs, c->px, M, DP, st));
  AttnParams ap;
  std::memset(&ap, 0, sizeof(ap));
  ap.q = c->pq;
  ap.q_ld = NQH * HD;
  ap.ca = dargs;
  ap.n_suf = 0;
  ap.nq = P;
  ap.n_splits = attn_splits(B, P, attn_keys(P, 0), c->sm_count, &ap.keys_per_split);
  ap.opart = c->popart;
  ap.mlpart = c->pmlpart;
  ap.out = c->po;
  ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)HD));
  ap.ctl = c->ctl;
  for (int l = 0; l < L; ++l) {
    CKN(launch_rmsnorm(c->px, c->pop, M, DP, eps, st));
    CKN(gemm_launch(c->tm_pwqkv, l * 2560, c->tm_pop, M, 2560, DP, c->pacc, c->tmo_pqkv, 2560, nullptr, false, c->ctl,
                    c->sm_count, st));
    CKN(launch_pf_qkv_post(c->pacc, dargs, l, P, c->rope_cos, c->rope_sin, c->rope_rows, c->pq, M, c->ctl, st));
    if (l == L - 1) break;  // the last layer only provides K/V to the expert
    ap.layer = l;
    CKN(attn_launch(ap, B, st));
    if (ap.n_splits > 1) ++n;
    CKN(gemm_launch(c->tm_pwo, l * DP, c->tm_po, M, DP, NQH * HD, c->px, c->tmo_px, DP, nullptr, true, c->ctl,
                    c->sm_count, st));
    CKN(launch_rmsnorm(c->px, c->pop, M, DP, eps, st));
    if (glu) {
      CKN(gemm_launch_glu(c->tm_pwgu64, l * 2 * FP, c->tm_pop, M, FP, DP, c->tm_pmb.m[0], nullptr, nullptr, c->ctl,
                          c->sm_count, st));
    } else {
      CKN(gemm_launch(c->tm_pwgu, l * 2 * FP, c->tm_pop, M, 2 * FP, DP, c->pacc, c->tmo_pgu, 2 * FP, nullptr, false,
                      c->ctl, c->sm_count, st));
      CKN(launch_gelu_mul(c->pacc, nullptr, nullptr, c->pmb, M, FP, st));
    }
    CKN(gemm_launch(c->tm_pwd, l * DP, c->tm_pmb, M, DP, FP, c->px, c->tmo_px, DP, nullptr, true, c->ctl, c->sm_count, st));
  }
  *kernels = n;
  return cudaSuccess;
}

rtvla_status capture(rtvla_ctx *c, bool prefill, int B, int P, GraphEntry *out) {
  int n = 0;
  cudaGraph_t g = nullptr;
  if (cudaStreamBeginCapture(c->cap_stream, cudaStreamCaptureModeThreadLocal) != cudaSuccess) return RTVLA_ERR_CUDA;
  cudaError_t e = prefill ? enqueue_prefill(c, c->args_pf, B, P, c->cap_stream, &n)
                          : enqueue_denoise(c, c->args_dn, B, P, c->cap_stream, nullptr, c->S - 1, &n);
  cudaError_t e2 = cudaStreamEndCapture(c->cap_stream, &g);
  if (e != cudaSuccess || e2 != cudaSuccess || !g) {
    if (g) cudaGraphDestroy(g);
    cudaGetLastError();
    return RTVLA_ERR_CUDA;
  }
  cudaGraphExec_t ex = nullptr;
  e = cudaGraphInstantiate(&ex, g, 0);
  cudaGraphDestroy(g);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return RTVLA_ERR_CUDA;
  }
  out->exec = ex;
  out->kernels = n;
  return RTVLA_OK;
}

bool use_persistent(const rtvla_ctx *c, int batch) {
  if (c->engine == RTVLA_ENGINE_LAYERED) return false;
  return c->pers_ok && batch == 1;
}

cudaError_t launch_persistent(rtvla_ctx *c, CallArgs *dargs, const rtvla_kv *kv, cudaStream_t st,
                              float *trace = nullptr, int trace_step = -1) {
  const int cap = kv->prefix_cap;
  c->pk_cache_k = kv->k;
  c->pk_cache_v = kv->v;
  PersistParams p;
  std::memset(&p, 0, sizeof(p));
  p.ca = dargs;
  p.bar = reinterpret_cast<unsigned int *>(reinterpret_cast<char *>(dargs) + offsetof(CallArgs, bar_count));
  static_assert(offsetof(CallArgs, bar_count) % 128 == 0, "barrier counters must start a 128-byte line");
  p.L = c->L;
  p.S = c->S;
  p.C = c->C;
  p.final_norm = c->cfg.final_norm;
  p.eps = c->cfg.rms_eps;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)HD));
  persistent_attn_plan(cap, c->C, c->sm_count, &p.attn_splits, &p.attn_cps);
  p.ca_cap = cap;
  // this call's prefix cache (batch 1): [L * cap][256] bf16, 32-key x 64-column boxes
  if (!make_map(&c->pmaps.l_kc, c->pk_cache_k, (uint64_t)c->L * cap, HD, 32) ||
      !make_map(&c->pmaps.l_vc, c->pk_cache_v, (uint64_t)c->L * cap, HD, 32))
    return cudaErrorInvalidValue;
  p.w_in = c->w_in;
  p.b_in = c->b_in;
  p.w_out = c->w_out;
  p.b_out = c->b_out;
  p.s1p_attn = c->s1p_attn;
  p.gate_attn = c->gate_attn;
  p.s1p_ffn = c->s1p_ffn;
  p.gate_ffn = c->gate_ffn;
  p.bias_qkv = c->bias_qkv;
  p.bias_gu = c->bias_gu;
  p.s1p_fin = c->s1p_fin;
  p.shift_fin = c->shift_fin;
  p.rope_cos = c->rope_cos;
  p.rope_sin = c->rope_sin;
  p.x = c->x;
  p.h = c->h;
  p.opart = c->pk_opart;
  p.mlpart = c->pk_mlpart;
  p.acc_qkv = c->acc_qkv;
  p.acc_gu = c->acc_gu;
  p.ss_attn = c->ss_attn;
  p.ss_ffn = c->ss_ffn;
  p.o = c->o;
  p.qb = c->q;
  p.ks = c->ks;
  p.vs = c->vs;
  p.ctl = c->ctl;
  p.stamps = c->pk_stamps;
  p.max_phases = c->pk_max_phases;
  p.trace = trace;
  p.trace_step = trace_step;
  if (c->variant == RTVLA_VARIANT_PI0) {
    p.pi0 = 1;
    p.w_fold = c->pi_wfold;
    p.c_tab = c->pi_ctab;
    p.b_ato = c->pi_bato;
    p.b_st = c->pi_bst;
    p.w_ato = c->pi_wato;
    p.w_st = c->pi_wst;
    p.op_ato = c->op;
  }
  return persistent_launch(c->pmaps, p, c->sm_count, st);
}

rtvla_status build_tables(rtvla_ctx *c, const rtvla_weights *w) {
  const int L = c->L, S = c->S;
  // time MLP in fp64 on the host: cond_k = SiLU(W_out SiLU(W_in e(t_k) + b_in) + b_out)
  std::vector<double> wi = d2h_bf16(w->time_in_w, (size_t)D * D), bi = d2h_bf16(w->time_in_b, D);
  std::vector<double> wo = d2h_bf16(w->time_out_w, (size_t)D * D), bo = d2h_bf16(w->time_out_b, D);
  if (wi.empty() || bi.empty() || wo.empty() || bo.empty()) return RTVLA_ERR_CUDA;
  std::vector<double> cond((size_t)S * D), e(D), hid(D);
  for (int k = 0; k < S; ++k) {
    const double t = 1.0 - (double)k / S;
    const int half = D / 2;
    for (int i = 0; i < half; ++i) {
      const double period = 4e-3 * std::pow(4.0 / 4e-3, (double)i / (half - 1));
      const double ang = 2.0 * M_PI * t / period;
      e[i] = std::sin(ang);
      e[i + half] = std::cos(ang);
    }
    for (int i = 0; i < D; ++i) {
      double a = bi[i];
      for (int j = 0; j < D; ++j) a += wi[(size_t)i * D + j] * e[j];
      hid[i] = silu_d(a);
    }
    for (int i = 0; i < D; ++i) {
      double a = bo[i];
      for (int j = 0; j < D; ++j) a += wo[(size_t)i * D + j] * hid[j];
      cond[(size_t)k * D + i] = silu_d(a);
    }
  }
  double *d_cond = dalloc<double>(c, (size_t)S * D);
  double *d_mod = dalloc<double>(c, (size_t)S * 8192);
  double *d_shift = dalloc<double>(c, (size_t)S * D);
  if (!d_cond || !d_mod || !d_shift) return RTVLA_ERR_OOM;
  if (cudaMemcpy(d_cond, cond.data(), cond.size() * 8, cudaMemcpyHostToDevice) != cudaSuccess) return RTVLA_ERR_CUDA;

  std::vector<double> mod((size_t)S * 3 * D), shift((size_t)S * D), big((size_t)S * 8192);
  std::vector<float> s1pA((size_t)S * L * D), gA((size_t)S * L * D), s1pF((size_t)S * L * D), gF((size_t)S * L * D);
  std::vector<float> bq((size_t)S * L * 2560), bg((size_t)S * L * 2 * F);
  for (int l = 0; l < L; ++l) {
    for (int which = 0; which < 2; ++which) {
      const void *aw = which == 0 ? w->ada_attn_w[l] : w->ada_ffn_w[l];
      const void *ab = which == 0 ? w->ada_attn_b[l] : w->ada_ffn_b[l];
      if (launch_rows_dot_f64(static_cast<const bf16 *>(aw), 3 * D, D, d_cond, S, static_cast<const bf16 *>(ab), d_mod,
                              0) != cudaSuccess)
        return RTVLA_ERR_CUDA;
      if (cudaMemcpy(mod.data(), d_mod, mod.size() * 8, cudaMemcpyDeviceToHost) != cudaSuccess) return RTVLA_ERR_CUDA;
      float *s1p = which == 0 ? s1pA.data() : s1pF.data();
      float *gt = which == 0 ? gA.data() : gF.data();
      for (int k = 0; k < S; ++k)
        for (int d = 0; d < D; ++d) {
          const size_t o = ((size_t)k * L + l) * D + d;
          s1p[o] = (float)(1.0 + mod[(size_t)k * 3 * D + d]);
          shift[(size_t)k * D + d] = mod[(size_t)k * 3 * D + D + d];
          gt[o] = (float)mod[(size_t)k * 3 * D + 2 * D + d];
        }
      // shift @ W^T: the AdaRMS shift pushed through the next GEMM as a bias
      if (cudaMemcpy(d_shift, shift.data(), shift.size() * 8, cudaMemcpyHostToDevice) != cudaSuccess)
        return RTVLA_ERR_CUDA;
      const int R = which == 0 ? 2560 : 2 * F;
      const bf16 *W = which == 0 ? c->w_qkv + (size_t)l * 2560 * D : c->w_gu + (size_t)l * 2 * F * D;
      if (launch_rows_dot_f64(W, R, D, d_shift, S, nullptr, d_mod, 0) != cudaSuccess) return RTVLA_ERR_CUDA;
      if (cudaMemcpy(big.data(), d_mod, (size_t)S * R * 8, cudaMemcpyDeviceToHost) != cudaSuccess)
        return RTVLA_ERR_CUDA;
      float *bt = which == 0 ? bq.data() : bg.data();
      for (int k = 0; k < S; ++k)
        for (int j = 0; j < R; ++j) bt[((size_t)k * L + l) * R + j] = (float)big[(size_t)k * R + j];
    }
  }
  std::vector<float> s1pfin((size_t)S * D, 1.0f), shfin((size_t)S * D, 0.0f);
  if (c->cfg.final_norm) {
    if (launch_rows_dot_f64(static_cast<const bf16 *>(w->ada_final_w), 3 * D, D, d_cond, S,
                            static_cast<const bf16 *>(w->ada_final_b), d_mod, 0) != cudaSuccess)
      return RTVLA_ERR_CUDA;
    if (cudaMemcpy(mod.data(), d_mod, mod.size() * 8, cudaMemcpyDeviceToHost) != cudaSuccess) return RTVLA_ERR_CUDA;
    for (int k = 0; k < S; ++k)
      for (int d = 0; d < D; ++d) {
        s1pfin[(size_t)k * D + d] = (float)(1.0 + mod[(size_t)k * 3 * D + d]);
        shfin[(size_t)k * D + d] = (float)mod[(size_t)k * 3 * D + D + d];
      }
  }
  struct {
    float *dst;
    const std::vector<float> *src;
  } up[] = {{c->s1p_attn, &s1pA}, {c->gate_attn, &gA}, {c->s1p_ffn, &s1pF}, {c->gate_ffn, &gF},
            {c->bias_qkv, &bq},   {c->bias_gu, &bg},   {c->s1p_fin, &s1pfin}, {c->shift_fin, &shfin}};
  for (auto &u : up)
    if (cudaMemcpy(u.dst, u.src->data(), u.src->size() * 4, cudaMemcpyHostToDevice) != cudaSuccess)
      return RTVLA_ERR_CUDA;

  return RTVLA_OK;
}

// The π0 tables ("Running VLAs at Real-time Speed" summary, "How"): plain RMSNorm is the
// AdaRMS form with scale = w, shift = 0 and gate = 1 (so the same kernels run it); the
// action-time MLP's first linear is folded with action_in_proj, W_fold = W_in[:, :D] W_a, and
// its 10 time rows become c_k = W_in[:, :D] b_a + W_in[:, D:] SinEmb(t_k) + b_in (fp64 on the
// host, rounded once to fp32).
rtvla_status build_tables_pi0(rtvla_ctx *c, const rtvla_weights *w) {
  const int L = c->L, S = c->S;
  std::vector<float> s1pA((size_t)S * L * D), s1pF((size_t)S * L * D), ones((size_t)S * L * D, 1.0f);
  for (int l = 0; l < L; ++l) {
    std::vector<double> g1 = d2h_bf16(w->ln1[l], D), g2 = d2h_bf16(w->ln2[l], D);
    if (g1.empty() || g2.empty()) return RTVLA_ERR_CUDA;
    for (int k = 0; k < S; ++k)
      for (int d = 0; d < D; ++d) {
        s1pA[((size_t)k * L + l) * D + d] = (float)(1.0 + g1[d]);
        s1pF[((size_t)k * L + l) * D + d] = (float)(1.0 + g2[d]);
      }
  }
  std::vector<double> gfin = d2h_bf16(w->final_ln, D);
  if (gfin.empty()) return RTVLA_ERR_CUDA;
  std::vector<float> s1pfin((size_t)S * D), shfin((size_t)S * D, 0.0f);
  for (int k = 0; k < S; ++k)
    for (int d = 0; d < D; ++d) s1pfin[(size_t)k * D + d] = (float)(1.0 + gfin[d]);
  std::vector<float> zq((size_t)S * L * 2560, 0.0f), zg((size_t)S * L * 2 * F, 0.0f);
  struct {
    float *dst;
    const std::vector<float> *src;
  } up[] = {{c->s1p_attn, &s1pA}, {c->gate_attn, &ones}, {c->s1p_ffn, &s1pF}, {c->gate_ffn, &ones},
            {c->bias_qkv, &zq},   {c->bias_gu, &zg},     {c->s1p_fin, &s1pfin}, {c->shift_fin, &shfin}};
  for (auto &u : up)
    if (cudaMemcpy(u.dst, u.src->data(), u.src->size() * 4, cudaMemcpyHostToDevice) != cudaSuccess)
      return RTVLA_ERR_CUDA;
  // fold and time table
  std::vector<double> wi = d2h_bf16(w->action_time_in_w, (size_t)D * 2 * D), bi = d2h_bf16(w->action_time_in_b, D);
  std::vector<double> wa = d2h_bf16(w->action_in_w, (size_t)D * A), ba = d2h_bf16(w->action_in_b, D);
  if (wi.empty() || bi.empty() || wa.empty() || ba.empty()) return RTVLA_ERR_CUDA;
  std::vector<float> fold((size_t)D * A), tab((size_t)S * D);
  std::vector<double> acc(A), e(D);
  for (int n = 0; n < D; ++n) {
    std::fill(acc.begin(), acc.end(), 0.0);
    for (int i = 0; i < D; ++i) {
      const double v = wi[(size_t)n * 2 * D + i];
      for (int a = 0; a < A; ++a) acc[a] += v * wa[(size_t)i * A + a];
    }
    for (int a = 0; a < A; ++a) fold[(size_t)n * A + a] = (float)acc[a];
  }
  for (int k = 0; k < S; ++k) {
    const double t = 1.0 - (double)k / S;
    const int half = D / 2;
    for (int i = 0; i < half; ++i) {
      const double period = 4e-3 * std::pow(4.0 / 4e-3, (double)i / (half - 1));
      const double ang = 2.0 * M_PI * t / period;
      e[i] = std::sin(ang);
      e[i + half] = std::cos(ang);
    }
    for (int n = 0; n < D; ++n) {
      double v = bi[n];
      for (int i = 0; i < D; ++i) v += wi[(size_t)n * 2 * D + i] * ba[i] + wi[(size_t)n * 2 * D + D + i] * e[i];
      tab[(size_t)k * D + n] = (float)v;
    }
  }
  if (cudaMemcpy(c->pi_wfold, fold.data(), fold.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(c->pi_ctab, tab.data(), tab.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess)
    return RTVLA_ERR_CUDA;
  return RTVLA_OK;
}

// RoPE cos/sin tables: angle = pos * theta^(-2i/256) in fp64, rounded once to fp32
rtvla_status build_rope(rtvla_ctx *c) {
  std::vector<float> rc((size_t)c->rope_rows * 128), rs((size_t)c->rope_rows * 128);
  for (int p = 0; p < c->rope_rows; ++p)
    for (int i = 0; i < 128; ++i) {
      const double ang = (double)p * std::pow((double)c->cfg.rope_theta, -2.0 * i / HD);
      rc[(size_t)p * 128 + i] = (float)std::cos(ang);
      rs[(size_t)p * 128 + i] = (float)std::sin(ang);
    }
  if (cudaMemcpy(c->rope_cos, rc.data(), rc.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(c->rope_sin, rs.data(), rs.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess)
    return RTVLA_ERR_CUDA;
  return RTVLA_OK;
}

size_t max_attn_partials(int Bmax, int nq, int keys, int sm) {
  size_t best = 0;
  for (int B = 1; B <= Bmax; ++B) {
    int kps;
    const int sp = attn_splits(B, nq, keys, sm, &kps);
    if (sp > 1) {
      const size_t v = (size_t)B * sp * nq;
      if (v > best) best = v;
    }
  }
  return best;
}

bool weights_present(const rtvla_weights *w, const rtvla_config *cfg) {
  const bool pi0 = cfg->variant == RTVLA_VARIANT_PI0;
  if (!w->action_in_w || !w->action_in_b || !w->action_out_w || !w->action_out_b) return false;
  if (!w->wq || !w->wk || !w->wv || !w->wo || !w->wg || !w->wu || !w->wd) return false;
  for (int l = 0; l < cfg->n_layers; ++l)
    if (!w->wq[l] || !w->wk[l] || !w->wv[l] || !w->wo[l] || !w->wg[l] || !w->wu[l] || !w->wd[l]) return false;
  if (pi0) {
    if (!w->state_w || !w->state_b || !w->action_time_in_w || !w->action_time_in_b || !w->action_time_out_w ||
        !w->action_time_out_b || !w->ln1 || !w->ln2 || !w->final_ln)
      return false;
    for (int l = 0; l < cfg->n_layers; ++l)
      if (!w->ln1[l] || !w->ln2[l]) return false;
  } else {
    if (!w->time_in_w || !w->time_in_b || !w->time_out_w || !w->time_out_b) return false;
    if (!w->ada_attn_w || !w->ada_attn_b || !w->ada_ffn_w || !w->ada_ffn_b) return false;
    for (int l = 0; l < cfg->n_layers; ++l)
      if (!w->ada_attn_w[l] || !w->ada_attn_b[l] || !w->ada_ffn_w[l] || !w->ada_ffn_b[l]) return false;
    if (cfg->final_norm && (!w->ada_final_w || !w->ada_final_b)) return false;
  }
  if (cfg->has_prefill) {
    if (!w->pf_ln1 || !w->pf_wq || !w->pf_wk || !w->pf_wv || !w->pf_wo || !w->pf_ln2 || !w->pf_wg || !w->pf_wu ||
        !w->pf_wd)
      return false;
    for (int l = 0; l < cfg->n_layers; ++l)
      if (!w->pf_ln1[l] || !w->pf_wq[l] || !w->pf_wk[l] || !w->pf_wv[l] || !w->pf_wo[l] || !w->pf_ln2[l] ||
          !w->pf_wg[l] || !w->pf_wu[l] || !w->pf_wd[l])
        return false;
  }
  return true;
}

rtvla_status create_impl(rtvla_ctx *c, const rtvla_weights *w) {
  const int L = c->L, S = c->S, C = c->C;
  if (cudaGetDevice(&c->device) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess)
    return RTVLA_ERR_CUDA;
  if (!get_encoder()) return RTVLA_ERR_CUDA;
  if (gemm_init_attributes() != cudaSuccess || attn_init_attributes() != cudaSuccess ||
      gemm2_init_attributes(c->sm_count) != cudaSuccess)
    return RTVLA_ERR_CUDA;
  if (cudaStreamCreateWithFlags(&c->cap_stream, cudaStreamNonBlocking) != cudaSuccess) return RTVLA_ERR_CUDA;

  // ---- weights: Q|K|V stacked, gate|up stacked, layers stacked (one tensor map each)
  c->w_qkv = dalloc<bf16>(c, (size_t)L * 2560 * D);
  c->w_o = dalloc<bf16>(c, (size_t)L * D * NQH * HD);
  c->w_gu = dalloc<bf16>(c, (size_t)L * 2 * F * D);
  c->w_d = dalloc<bf16>(c, (size_t)L * D * F);
  c->w_in = dalloc<bf16>(c, (size_t)D * A);
  c->b_in = dalloc<float>(c, D);
  c->w_out = dalloc<float>(c, (size_t)A * D);
  c->b_out = dalloc<float>(c, A);
  if (!c->w_qkv || !c->w_o || !c->w_gu || !c->w_d || !c->w_in || !c->b_in || !c->w_out || !c->b_out)
    return RTVLA_ERR_OOM;
  const cudaMemcpyKind dd = cudaMemcpyDeviceToDevice;
  for (int l = 0; l < L; ++l) {
    bf16 *qkv = c->w_qkv + (size_t)l * 2560 * D;
    bf16 *gu = c->w_gu + (size_t)l * 2 * F * D;
    if (cudaMemcpy(qkv, w->wq[l], (size_t)2048 * D * 2, dd) != cudaSuccess ||
        cudaMemcpy(qkv + (size_t)2048 * D, w->wk[l], (size_t)HD * D * 2, dd) != cudaSuccess ||
        cudaMemcpy(qkv + (size_t)2304 * D, w->wv[l], (size_t)HD * D * 2, dd) != cudaSuccess ||
        cudaMemcpy(c->w_o + (size_t)l * D * 2048, w->wo[l], (size_t)D * 2048 * 2, dd) != cudaSuccess ||
        cudaMemcpy(gu, w->wg[l], (size_t)F * D * 2, dd) != cudaSuccess ||
        cudaMemcpy(gu + (size_t)F * D, w->wu[l], (size_t)F * D * 2, dd) != cudaSuccess ||
        cudaMemcpy(c->w_d + (size_t)l * D * F, w->wd[l], (size_t)D * F * 2, dd) != cudaSuccess)
      return RTVLA_ERR_CUDA;
  }
  const double dt = -1.0 / S;  // Euler step folded into action_out_proj
  if (cudaMemcpy(c->w_in, w->action_in_w, (size_t)D * A * 2, dd) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (c->variant == RTVLA_VARIANT_PI0) {
    c->pi_wfold = dalloc<float>(c, (size_t)D * A);
    c->pi_ctab = dalloc<float>(c, (size_t)S * D);
    c->pi_wato = dalloc<bf16>(c, (size_t)D * D);
    c->pi_bato = dalloc<float>(c, D);
    c->pi_wst = dalloc<bf16>(c, (size_t)D * A);
    c->pi_bst = dalloc<float>(c, D);
    if (!c->pi_wfold || !c->pi_ctab || !c->pi_wato || !c->pi_bato || !c->pi_wst || !c->pi_bst) return RTVLA_ERR_OOM;
    if (cudaMemcpy(c->pi_wato, w->action_time_out_w, (size_t)D * D * 2, dd) != cudaSuccess ||
        cudaMemcpy(c->pi_wst, w->state_w, (size_t)D * A * 2, dd) != cudaSuccess ||
        launch_scale_to_f32(static_cast<const bf16 *>(w->action_time_out_b), D, 1.0, c->pi_bato, 0) != cudaSuccess ||
        launch_scale_to_f32(static_cast<const bf16 *>(w->state_b), D, 1.0, c->pi_bst, 0) != cudaSuccess)
      return RTVLA_ERR_CUDA;
  }
  if (launch_scale_to_f32(static_cast<const bf16 *>(w->action_in_b), D, 1.0, c->b_in, 0) != cudaSuccess ||
      launch_scale_to_f32(static_cast<const bf16 *>(w->action_out_w), A * D, dt, c->w_out, 0) != cudaSuccess ||
      launch_scale_to_f32(static_cast<const bf16 *>(w->action_out_b), A, dt, c->b_out, 0) != cudaSuccess)
    return RTVLA_ERR_CUDA;

  // ---- tables
  c->rope_rows = c->Pmax + C + 1;
  c->s1p_attn = dalloc<float>(c, (size_t)S * L * D);
  c->gate_attn = dalloc<float>(c, (size_t)S * L * D);
  c->s1p_ffn = dalloc<float>(c, (size_t)S * L * D);
  c->gate_ffn = dalloc<float>(c, (size_t)S * L * D);
  c->bias_qkv = dalloc<float>(c, (size_t)S * L * 2560);
  c->bias_gu = dalloc<float>(c, (size_t)S * L * 2 * F);
  c->s1p_fin = dalloc<float>(c, (size_t)S * D);
  c->shift_fin = dalloc<float>(c, (size_t)S * D);
  c->rope_cos = dalloc<float>(c, (size_t)c->rope_rows * 128);
  c->rope_sin = dalloc<float>(c, (size_t)c->rope_rows * 128);
  if (!c->s1p_attn || !c->gate_attn || !c->s1p_ffn || !c->gate_ffn || !c->bias_qkv || !c->bias_gu || !c->s1p_fin ||
      !c->shift_fin || !c->rope_cos || !c->rope_sin)
    return RTVLA_ERR_OOM;
  rtvla_status st = c->variant == RTVLA_VARIANT_PI0 ? build_tables_pi0(c, w) : build_tables(c, w);
  if (st != RTVLA_OK) return st;
  st = build_rope(c);
  if (st != RTVLA_OK) return st;

  // ---- prefix-pass weights, Gemma RMSNorm (1 + w) folded into the following projection
  if (c->cfg.has_prefill) {
    c->pw_qkv = dalloc<bf16>(c, (size_t)L * 2560 * DP);
    c->pw_o = dalloc<bf16>(c, (size_t)L * DP * NQH * HD);
    c->pw_gu = dalloc<bf16>(c, (size_t)L * 2 * FP * DP);
    c->pw_d = dalloc<bf16>(c, (size_t)L * DP * FP);
    if (!c->pw_qkv || !c->pw_o || !c->pw_gu || !c->pw_d) return RTVLA_ERR_OOM;
    for (int l = 0; l < L; ++l) {
      bf16 *qkv = c->pw_qkv + (size_t)l * 2560 * DP;
      bf16 *gu = c->pw_gu + (size_t)l * 2 * FP * DP;
      const bf16 *g1 = static_cast<const bf16 *>(w->pf_ln1[l]);
      const bf16 *g2 = static_cast<const bf16 *>(w->pf_ln2[l]);
      if (launch_fold_cols(static_cast<const bf16 *>(w->pf_wq[l]), 2048, DP, g1, qkv, 0) != cudaSuccess ||
          launch_fold_cols(static_cast<const bf16 *>(w->pf_wk[l]), HD, DP, g1, qkv + (size_t)2048 * DP, 0) !=
              cudaSuccess ||
          launch_fold_cols(static_cast<const bf16 *>(w->pf_wv[l]), HD, DP, g1, qkv + (size_t)2304 * DP, 0) !=
              cudaSuccess ||
          launch_fold_cols(static_cast<const bf16 *>(w->pf_wg[l]), FP, DP, g2, gu, 0) != cudaSuccess ||
          launch_fold_cols(static_cast<const bf16 *>(w->pf_wu[l]), FP, DP, g2, gu + (size_t)FP * DP, 0) !=
              cudaSuccess ||
          cudaMemcpy(c->pw_o + (size_t)l * DP * 2048, w->pf_wo[l], (size_t)DP * 2048 * 2, dd) != cudaSuccess ||
          cudaMemcpy(c->pw_d + (size_t)l * DP * FP, w->pf_wd[l], (size_t)DP * FP * 2, dd) != cudaSuccess)
        return RTVLA_ERR_CUDA;
    }
  }

  // ---- static activation buffers
  // rows are padded to a multiple of 256 so that every token-tile box stays inside the buffer
  c->Mmax = c->Bmax * C;
  const size_t M = ((size_t)c->Mmax + 255) / 256 * 256;
  c->x = dalloc<float>(c, M * A);
  c->h = dalloc<float>(c, M * D);
  c->r = dalloc<float>(c, M);
  c->acc_qkv = dalloc<float>(c, M * 2560);
  c->acc_gu = dalloc<float>(c, M * 2 * F);
  c->op = dalloc<bf16>(c, M * D);
  c->q = dalloc<bf16>(c, M * NQH * HD);
  c->ks = dalloc<bf16>(c, M * HD);
  c->vs = dalloc<bf16>(c, M * HD);
  c->o = dalloc<bf16>(c, M * NQH * HD);
  c->mb = dalloc<bf16>(c, M * F);
  const size_t parts = max_attn_partials(c->Bmax, C, attn_keys(c->Pmax, C), c->sm_count);
  c->opart = dalloc<float>(c, parts * NQH * HD);
  c->mlpart = dalloc<float>(c, parts * NQH * 2);
  if (!c->x || !c->h || !c->r || !c->acc_qkv || !c->acc_gu || !c->op || !c->q || !c->ks || !c->vs || !c->o ||
      !c->mb || !c->opart || !c->mlpart)
    return RTVLA_ERR_OOM;
  c->Mpmax = c->cfg.has_prefill ? c->Bmax * c->Pmax : 0;
  const size_t Mp = ((size_t)c->Mpmax + 255) / 256 * 256;
  if (c->cfg.has_prefill) {
    c->px = dalloc<float>(c, Mp * DP);
    c->pacc = dalloc<float>(c, Mp * 2 * FP);
    c->pop = dalloc<bf16>(c, Mp * DP);
    c->pq = dalloc<bf16>(c, Mp * NQH * HD);
    c->po = dalloc<bf16>(c, Mp * NQH * HD);
    c->pmb = dalloc<bf16>(c, Mp * FP);
    const size_t pparts = max_attn_partials(c->Bmax, c->Pmax, attn_keys(c->Pmax, 0), c->sm_count);
    c->popart = dalloc<float>(c, pparts * NQH * HD);
    c->pmlpart = dalloc<float>(c, pparts * NQH * 2);
    if (!c->px || !c->pacc || !c->pop || !c->pq || !c->po || !c->pmb || !c->popart || !c->pmlpart)
      return RTVLA_ERR_OOM;
    if (cudaMemset(c->pacc, 0, Mp * 2 * FP * 4) != cudaSuccess) return RTVLA_ERR_CUDA;
  }
  if (cudaMemset(c->acc_qkv, 0, M * 2560 * 4) != cudaSuccess || cudaMemset(c->acc_gu, 0, M * 2 * F * 4) != cudaSuccess)
    return RTVLA_ERR_CUDA;

  // ---- tensor maps (weights: 128-row boxes; activations: one map per token-tile height)
  bool ok = (c->variant != RTVLA_VARIANT_PI0 || make_map(&c->tm_wato, c->pi_wato, D, D, 128)) &&
            make_map(&c->tm_wqkv, c->w_qkv, (uint64_t)L * 2560, D, 128) &&
            make_map(&c->tm_wo, c->w_o, (uint64_t)L * D, NQH * HD, 128) &&
            make_map(&c->tm_wgu, c->w_gu, (uint64_t)L * 2 * F, D, 128) &&
            make_map(&c->tm_wgu64, c->w_gu, (uint64_t)L * 2 * F, D, 64) &&
            make_map(&c->tm_wd, c->w_d, (uint64_t)L * D, F, 128) && make_xmaps(&c->tm_op, c->op, M, D) &&
            make_xmaps(&c->tm_o, c->o, M, NQH * HD) && make_xmaps(&c->tm_mb, c->mb, M, F) &&
            make_map(&c->tm_q64, c->q, M, NQH * HD, 64) && make_map_f32(&c->tmo_qkv, c->acc_qkv, M, 2560, 128, false) &&
            make_map_f32(&c->tmo_h, c->h, M, D, 128, false) && make_map_f32(&c->tmo_gu, c->acc_gu, M, 2 * F, 128, false);
  if (c->cfg.has_prefill) {
    ok = ok && make_map(&c->tm_pwqkv, c->pw_qkv, (uint64_t)L * 2560, DP, 128) &&
         make_map(&c->tm_pwo, c->pw_o, (uint64_t)L * DP, NQH * HD, 128) &&
         make_map(&c->tm_pwgu, c->pw_gu, (uint64_t)L * 2 * FP, DP, 128) &&
         make_map(&c->tm_pwgu64, c->pw_gu, (uint64_t)L * 2 * FP, DP, 64) &&
         make_map(&c->tm_pwd, c->pw_d, (uint64_t)L * DP, FP, 128) &&
         make_xmaps(&c->tm_pop, c->pop, Mp, DP) && make_xmaps(&c->tm_po, c->po, Mp, NQH * HD) &&
         make_xmaps(&c->tm_pmb, c->pmb, Mp, FP) && make_map_f32(&c->tmo_pqkv, c->pacc, Mp, 2560, 128, false) &&
         make_map_f32(&c->tmo_px, c->px, Mp, DP, 128, false) && make_map_f32(&c->tmo_pgu, c->pacc, Mp, 2 * FP, 128, false);
  }
  if (!ok) return RTVLA_ERR_CUDA;

  // ---- persistent engine (batch 1, chunk <= 64): norm statistics and attention partials
  if (persistent_init_attributes() != cudaSuccess) return RTVLA_ERR_CUDA;
  c->pers_ok = C <= 64 && persistent_fits(c->sm_count);
  if (c->pers_ok) {
    const int sp = persistent_max_splits(c->sm_count);
    c->ss_attn = dalloc<float>(c, 64);
    c->ss_ffn = dalloc<float>(c, 64);
    c->pk_opart = dalloc<float>(c, (size_t)sp * NQH * 64 * HD);
    c->pk_mlpart = dalloc<float>(c, (size_t)sp * NQH * 64 * 2);
    if (!c->ss_attn || !c->ss_ffn || !c->pk_opart || !c->pk_mlpart) return RTVLA_ERR_OOM;
    PersistMaps &pm = c->pmaps;
    pm.w_qkv = c->tm_wqkv;
    pm.w_o = c->tm_wo;
    pm.w_gu = c->tm_wgu;
    pm.w_d = c->tm_wd;
    pm.l_o = c->tm_o.m[0];
    pm.l_q = c->tm_q64;
    if (!make_map_f32(&pm.r_qkv, c->acc_qkv, 64, 2560, 128, false) ||
        !make_map_f32(&pm.r_gu, c->acc_gu, 64, 2 * F, 128, false) || !make_map_f32(&pm.r_h, c->h, 64, D, 128, false) ||
        !make_map_f32_blocks(&pm.l_h, c->h, D, 4) || !make_map_f32_blocks(&pm.l_gu, c->acc_gu, 2 * F, 2) ||
        !make_map(&pm.l_ks, c->ks, 256, HD, 32) || !make_map(&pm.l_vs, c->vs, 256, HD, 32))
      return RTVLA_ERR_CUDA;
    if (std::getenv("RTVLA_PHASE_STAMPS")) {
      c->pk_max_phases = c->S * (7 * c->L + 1) + 2;
      c->pk_stamps = dalloc<unsigned long long>(c, (size_t)c->sm_count * c->pk_max_phases * 8);
      if (!c->pk_stamps) return RTVLA_ERR_OOM;
      cudaMemset(c->pk_stamps, 0, (size_t)c->sm_count * c->pk_max_phases * 8 * 8);
    }
  }

  // ---- control block and argument blocks
  c->ctl = dalloc<DevCtl>(c, 1);
  c->args_dn = dalloc<CallArgs>(c, 1);
  c->args_pf = dalloc<CallArgs>(c, 1);
  c->args_tr = dalloc<CallArgs>(c, 1);
  if (!c->ctl || !c->args_dn || !c->args_pf || !c->args_tr) return RTVLA_ERR_OOM;
  DevCtl hc;
  std::memset(&hc, 0, sizeof(hc));
  hc.timeout_ns = 2000000000ull;
  if (const char *env = std::getenv("RTVLA_WAIT_TIMEOUT_US")) {
    const long long us = std::atoll(env);
    if (us > 0) hc.timeout_ns = (unsigned long long)us * 1000ull;
  }
  if (cudaMemcpy(c->ctl, &hc, sizeof(hc), cudaMemcpyHostToDevice) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return RTVLA_ERR_CUDA;
  return RTVLA_OK;
}

}  // namespace

// =======================================================================================
// C ABI

extern "C" {

const char *rtvla_status_string(rtvla_status s) {
  switch (s) {
    case RTVLA_OK: return "ok";
    case RTVLA_ERR_INVALID_ARG: return "invalid argument";
    case RTVLA_ERR_SHAPE: return "shape exceeds the context's capacity";
    case RTVLA_ERR_MASK_NOT_PREFIX: return "pad mask is not a prefix of valid tokens";
    case RTVLA_ERR_OOM: return "out of device memory";
    case RTVLA_ERR_CUDA: return "CUDA runtime error";
    case RTVLA_ERR_DEVICE_TIMEOUT: return "a bounded device wait expired";
    case RTVLA_ERR_UNSUPPORTED: return "unsupported model shape or engine";
    case RTVLA_ERR_DEVICE_BOUNDS: return "a valid length exceeded its buffer";
    case RTVLA_ERR_GUARD_OVERWRITE: return "a guard band around a library buffer was overwritten";
  }
  return "unknown status";
}

size_t rtvla_kv_bytes(const rtvla_config *cfg, int batch, int prefix_cap) {
  if (!cfg || batch < 1 || prefix_cap < 1 || cfg->n_layers < 1 || cfg->head_dim < 1 || cfg->n_kv_heads < 1) return 0;
  return 2ull * (size_t)cfg->n_layers * batch * prefix_cap * cfg->n_kv_heads * cfg->head_dim * 2ull;
}

rtvla_status rtvla_create(const rtvla_weights *w, const rtvla_config *cfg, rtvla_ctx **out) {
  if (!w || !cfg || !out) return RTVLA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!valid_cfg(cfg)) return RTVLA_ERR_INVALID_ARG;
  if (!supported_cfg(cfg)) return RTVLA_ERR_UNSUPPORTED;
  if (!weights_present(w, cfg)) return RTVLA_ERR_INVALID_ARG;
  rtvla_ctx *c = new rtvla_ctx();
  c->cfg = *cfg;
  c->L = cfg->n_layers;
  c->S = cfg->n_steps;
  c->variant = cfg->variant;
  c->first = cfg->variant == RTVLA_VARIANT_PI0 ? 1 : 0;
  if (c->variant == RTVLA_VARIANT_PI0) c->cfg.final_norm = 1;  // π0 ends in an RMSNorm
  c->Ca = cfg->chunk;
  c->C = cfg->chunk + c->first;
  c->Bmax = cfg->max_batch;
  c->Pmax = cfg->max_prefix;
  c->engine = cfg->engine;
  if (const char *env = std::getenv("RTVLA_CHECKED")) c->checked = std::atoi(env) != 0;
  if (const char *env = std::getenv("RTVLA_DEVICE_MEMORY_CAP")) c->mem_cap = (size_t)std::strtoull(env, nullptr, 10);
  rtvla_status st = create_impl(c, w);
  if (st == RTVLA_OK && c->checked) {
    const size_t b = c->guards.size() * sizeof(GuardRegion);
    if (cudaMalloc(&c->d_guards, b) != cudaSuccess ||
        cudaMemcpy(c->d_guards, c->guards.data(), b, cudaMemcpyHostToDevice) != cudaSuccess)
      st = RTVLA_ERR_CUDA;
  }
  if (st != RTVLA_OK) {
    cudaGetLastError();
    free_all(c);
    return st;
  }
  *out = c;
  return RTVLA_OK;
}

void rtvla_destroy(rtvla_ctx *c) {
  if (!c) return;
  cudaDeviceSynchronize();
  if (c->pk_stamps) {
    // debug aid: raw phase timestamps of the last persistent launch, [grid][phases][8] u64
    const char *path = std::getenv("RTVLA_PHASE_STAMPS");
    const size_t n = (size_t)c->sm_count * c->pk_max_phases * 8;
    std::vector<unsigned long long> h(n);
    if (path && cudaMemcpy(h.data(), c->pk_stamps, n * 8, cudaMemcpyDeviceToHost) == cudaSuccess) {
      if (FILE *f = std::fopen(path, "wb")) {
        const int hdr[2] = {c->sm_count, c->pk_max_phases};
        std::fwrite(hdr, sizeof(hdr), 1, f);
        std::fwrite(h.data(), 8, n, f);
        std::fclose(f);
      }
    }
  }
  free_all(c);
}

static rtvla_status check_kv(rtvla_ctx *c, const rtvla_kv *kv) {
  if (!kv || !kv->k || !kv->v || !kv->valid_len) return RTVLA_ERR_INVALID_ARG;
  if (kv->batch < 1 || kv->prefix_cap < 1) return RTVLA_ERR_INVALID_ARG;
  if (kv->batch > c->Bmax || kv->prefix_cap > c->Pmax) return RTVLA_ERR_SHAPE;
  return RTVLA_OK;
}

static CallArgs host_args(const rtvla_kv *kv) {
  CallArgs a;
  std::memset(&a, 0, sizeof(a));
  a.kv_k = static_cast<const bf16 *>(kv->k);
  a.kv_v = static_cast<const bf16 *>(kv->v);
  a.valid_len = kv->valid_len;
  a.batch = kv->batch;
  a.cap = kv->prefix_cap;
  return a;
}

static rtvla_status sample_impl(rtvla_ctx *c, const float *noise, const float *state, const rtvla_kv *kv,
                                float *actions_out, void *stream) {
  rtvla_status s = check_kv(c, kv);
  if (s != RTVLA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CallArgs a = host_args(kv);
  a.noise = noise;
  a.actions = actions_out;
  a.state = state;
  if (c->engine == RTVLA_ENGINE_PERSISTENT && !use_persistent(c, kv->batch)) return RTVLA_ERR_UNSUPPORTED;
  if (use_persistent(c, kv->batch)) {
    if (cudaMemcpyAsync(c->args_dn, &a, sizeof(a), cudaMemcpyHostToDevice, st) != cudaSuccess) return RTVLA_ERR_CUDA;
    if (launch_persistent(c, c->args_dn, kv, st) != cudaSuccess) {
      cudaGetLastError();
      return RTVLA_ERR_CUDA;
    }
    c->kernels_per_call[kv->batch] = 1;
    return RTVLA_OK;
  }
  const auto key = std::make_pair(kv->batch, kv->prefix_cap);
  auto it = c->graphs_dn.find(key);
  if (it == c->graphs_dn.end()) {
    GraphEntry g;
    s = capture(c, false, kv->batch, kv->prefix_cap, &g);
    if (s != RTVLA_OK) return s;
    it = c->graphs_dn.emplace(key, g).first;
  }
  if (cudaMemcpyAsync(c->args_dn, &a, sizeof(a), cudaMemcpyHostToDevice, st) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (cudaGraphLaunch(it->second.exec, st) != cudaSuccess) return RTVLA_ERR_CUDA;
  c->kernels_per_call[kv->batch] = it->second.kernels;
  return RTVLA_OK;
}

rtvla_status rtvla_sample_actions(rtvla_ctx *c, const float *noise, const rtvla_kv *kv, float *actions_out,
                                  void *stream) {
  if (!c || !noise || !actions_out) return RTVLA_ERR_INVALID_ARG;
  if (c->variant != RTVLA_VARIANT_PI05) return RTVLA_ERR_INVALID_ARG;  // π0 needs the state
  return sample_impl(c, noise, nullptr, kv, actions_out, stream);
}

rtvla_status rtvla_sample_actions_pi0(rtvla_ctx *c, const float *noise, const float *state, const rtvla_kv *kv,
                                      float *actions_out, void *stream) {
  if (!c || !noise || !state || !actions_out) return RTVLA_ERR_INVALID_ARG;
  if (c->variant != RTVLA_VARIANT_PI0) return RTVLA_ERR_UNSUPPORTED;
  return sample_impl(c, noise, state, kv, actions_out, stream);
}

rtvla_status rtvla_sample_actions_host(rtvla_ctx *c, const float *noise, const void *kv_k, const void *kv_v,
                                       const int32_t *valid_len, int batch, int prefix_cap, float *actions_out,
                                       void *stream) {
  if (!c || !noise || !kv_k || !kv_v || !valid_len || !actions_out) return RTVLA_ERR_INVALID_ARG;
  if (c->variant != RTVLA_VARIANT_PI05) return RTVLA_ERR_INVALID_ARG;  // π0 needs the state
  if (batch < 1 || prefix_cap < 1) return RTVLA_ERR_INVALID_ARG;
  if (batch > c->Bmax || prefix_cap > c->Pmax) return RTVLA_ERR_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t kv_elems = (size_t)c->L * batch * prefix_cap * HD;
  const size_t io = (size_t)batch * c->Ca * A;
  if (kv_elems > c->st_kv_elems) {
    if (c->st_k) cudaFree(c->st_k);
    if (c->st_v) cudaFree(c->st_v);
    c->st_k = c->st_v = nullptr;
    c->st_kv_elems = 0;
    if (cudaMalloc(&c->st_k, kv_elems * 2) != cudaSuccess || cudaMalloc(&c->st_v, kv_elems * 2) != cudaSuccess) {
      cudaGetLastError();
      return RTVLA_ERR_OOM;
    }
    c->st_kv_elems = kv_elems;
  }
  if (io > c->st_io_elems || batch > c->st_batch) {
    if (c->st_noise) cudaFree(c->st_noise);
    if (c->st_act) cudaFree(c->st_act);
    if (c->st_vl) cudaFree(c->st_vl);
    c->st_noise = c->st_act = nullptr;
    c->st_vl = nullptr;
    c->st_io_elems = 0;
    c->st_batch = 0;
    if (cudaMalloc(&c->st_noise, io * 4) != cudaSuccess || cudaMalloc(&c->st_act, io * 4) != cudaSuccess ||
        cudaMalloc(&c->st_vl, (size_t)batch * 4) != cudaSuccess) {
      cudaGetLastError();
      return RTVLA_ERR_OOM;
    }
    c->st_io_elems = io;
    c->st_batch = batch;
  }
  const cudaMemcpyKind hd = cudaMemcpyHostToDevice;
  if (cudaMemcpyAsync(c->st_noise, noise, io * 4, hd, st) != cudaSuccess ||
      cudaMemcpyAsync(c->st_k, kv_k, kv_elems * 2, hd, st) != cudaSuccess ||
      cudaMemcpyAsync(c->st_v, kv_v, kv_elems * 2, hd, st) != cudaSuccess ||
      cudaMemcpyAsync(c->st_vl, valid_len, (size_t)batch * 4, hd, st) != cudaSuccess)
    return RTVLA_ERR_CUDA;
  rtvla_kv kv;
  kv.k = c->st_k;
  kv.v = c->st_v;
  kv.valid_len = c->st_vl;
  kv.batch = batch;
  kv.prefix_cap = prefix_cap;
  rtvla_status s = rtvla_sample_actions(c, c->st_noise, &kv, c->st_act, stream);
  if (s != RTVLA_OK) return s;
  if (cudaMemcpyAsync(actions_out, c->st_act, io * 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return RTVLA_ERR_CUDA;
  return RTVLA_OK;
}

rtvla_status rtvla_prefill(rtvla_ctx *c, const void *prefix_embeds, const uint8_t *pad_mask, int batch,
                           int prefix_len, const rtvla_kv *kv_out, void *stream) {
  if (!c || !prefix_embeds || !pad_mask || !kv_out || !kv_out->k || !kv_out->v || !kv_out->valid_len)
    return RTVLA_ERR_INVALID_ARG;
  if (batch < 1 || prefix_len < 1 || kv_out->prefix_cap < 1) return RTVLA_ERR_INVALID_ARG;
  if (!c->cfg.has_prefill) return RTVLA_ERR_UNSUPPORTED;
  if (batch > c->Bmax || kv_out->batch != batch || prefix_len > kv_out->prefix_cap || prefix_len > c->Pmax)
    return RTVLA_ERR_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CallArgs a;
  std::memset(&a, 0, sizeof(a));
  a.kv_k = static_cast<const bf16 *>(kv_out->k);
  a.kv_v = static_cast<const bf16 *>(kv_out->v);
  a.valid_len = kv_out->valid_len;
  a.batch = batch;
  a.cap = kv_out->prefix_cap;
  a.embeds = static_cast<const bf16 *>(prefix_embeds);
  a.mask = pad_mask;
  a.kvo_k = static_cast<bf16 *>(kv_out->k);
  a.kvo_v = static_cast<bf16 *>(kv_out->v);
  a.valid_out = kv_out->valid_len;
  a.pf_len = prefix_len;
  const auto key = std::make_pair(batch, prefix_len * 65536 + kv_out->prefix_cap);
  auto it = c->graphs_pf.find(key);
  if (it == c->graphs_pf.end()) {
    GraphEntry g;
    rtvla_status s = capture(c, true, batch, prefix_len, &g);
    if (s != RTVLA_OK) return s;
    it = c->graphs_pf.emplace(key, g).first;
  }
  if (cudaMemcpyAsync(c->args_pf, &a, sizeof(a), cudaMemcpyHostToDevice, st) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (cudaGraphLaunch(it->second.exec, st) != cudaSuccess) return RTVLA_ERR_CUDA;
  return RTVLA_OK;
}

rtvla_status rtvla_sync_status(rtvla_ctx *c, void *stream) {
  if (!c) return RTVLA_ERR_INVALID_ARG;
  if (c->checked &&
      launch_check_guards(c->d_guards, (int)c->guards.size(), c->ctl, static_cast<cudaStream_t>(stream)) !=
          cudaSuccess) {
    cudaGetLastError();
    return RTVLA_ERR_CUDA;
  }
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return RTVLA_ERR_CUDA;
  }
  DevCtl h;
  if (cudaMemcpy(&h, c->ctl, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (h.err == 0) return RTVLA_OK;
  const int zero[2] = {0, 0};
  if (cudaMemcpy(c->ctl, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (h.err & DEVERR_TIMEOUT) return RTVLA_ERR_DEVICE_TIMEOUT;
  if (h.err & DEVERR_MASK) return RTVLA_ERR_MASK_NOT_PREFIX;
  if (h.err & DEVERR_GUARD) return RTVLA_ERR_GUARD_OVERWRITE;
  return RTVLA_ERR_DEVICE_BOUNDS;
}

rtvla_status rtvla_debug_plant_guard_fault(rtvla_ctx *c) {
  if (!c) return RTVLA_ERR_INVALID_ARG;
  if (!c->checked) return RTVLA_ERR_UNSUPPORTED;
  for (const GuardRegion &g : c->guards)
    if (g.base + GUARD_BYTES == reinterpret_cast<unsigned char *>(c->h)) {
      // the first byte past the end of the residual-stream buffer, as a kernel writing one
      // row too far would touch it
      if (cudaDeviceSynchronize() != cudaSuccess || cudaMemset(g.base + GUARD_BYTES + g.bytes, 0, 1) != cudaSuccess) {
        cudaGetLastError();
        return RTVLA_ERR_CUDA;
      }
      return RTVLA_OK;
    }
  return RTVLA_ERR_UNSUPPORTED;
}

static rtvla_status trace_impl(rtvla_ctx *c, const float *noise, const float *state, const rtvla_kv *kv, int step,
                               float *h_layers, void *stream) {
  rtvla_status s = check_kv(c, kv);
  if (s != RTVLA_OK) return s;
  if (step < 0 || step >= c->S) return RTVLA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CallArgs a = host_args(kv);
  a.noise = noise;
  a.actions = nullptr;
  a.state = state;
  if (c->engine == RTVLA_ENGINE_PERSISTENT && !use_persistent(c, kv->batch)) return RTVLA_ERR_UNSUPPORTED;
  if (cudaMemcpyAsync(c->args_tr, &a, sizeof(a), cudaMemcpyHostToDevice, st) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (use_persistent(c, kv->batch)) {
    // the engine rtvla_sample_actions would run: the persistent kernel, recording h at `step`
    if (launch_persistent(c, c->args_tr, kv, st, h_layers, step) != cudaSuccess) {
      cudaGetLastError();
      return RTVLA_ERR_CUDA;
    }
    return RTVLA_OK;
  }
  int n = 0;
  if (enqueue_denoise(c, c->args_tr, kv->batch, kv->prefix_cap, st, h_layers, step, &n) != cudaSuccess)
    return RTVLA_ERR_CUDA;
  return RTVLA_OK;
}

rtvla_status rtvla_debug_trace(rtvla_ctx *c, const float *noise, const rtvla_kv *kv, int step, float *h_layers,
                               void *stream) {
  if (!c || !noise || !h_layers) return RTVLA_ERR_INVALID_ARG;
  if (c->variant != RTVLA_VARIANT_PI05) return RTVLA_ERR_INVALID_ARG;
  return trace_impl(c, noise, nullptr, kv, step, h_layers, stream);
}

rtvla_status rtvla_debug_trace_pi0(rtvla_ctx *c, const float *noise, const float *state, const rtvla_kv *kv, int step,
                                   float *h_layers, void *stream) {
  if (!c || !noise || !state || !h_layers) return RTVLA_ERR_INVALID_ARG;
  if (c->variant != RTVLA_VARIANT_PI0) return RTVLA_ERR_UNSUPPORTED;
  return trace_impl(c, noise, state, kv, step, h_layers, stream);
}

int rtvla_kernels_per_call(rtvla_ctx *c, int batch) {
  if (!c) return -1;
  auto it = c->kernels_per_call.find(batch);
  return it == c->kernels_per_call.end() ? -1 : it->second;
}

rtvla_status rtvla_set_engine(rtvla_ctx *c, int engine) {
  if (!c || engine < 0 || engine > 2) return RTVLA_ERR_INVALID_ARG;
  c->engine = engine;
  return RTVLA_OK;
}

rtvla_status rtvla_set_wait_timeout_us(rtvla_ctx *c, long long us) {
  if (!c || us <= 0) return RTVLA_ERR_INVALID_ARG;
  const unsigned long long ns = (unsigned long long)us * 1000ull;
  if (cudaMemcpy(&c->ctl->timeout_ns, &ns, sizeof(ns), cudaMemcpyHostToDevice) != cudaSuccess) return RTVLA_ERR_CUDA;
  return RTVLA_OK;
}

}  // extern "C"

// =======================================================================================
// Allocation-free host-buffer call.
//
// Same computation as rtvla_sample_actions_host, for callers that must not allocate device
// memory once they are running (see include/rtvla.h).  The device staging that
// rtvla_sample_actions_host obtains with cudaMalloc on first use lives here in a fixed
// file-scope array instead; every GPU that loads this library holds that array until the
// process exits.

#define RTVLA_STATIC_STAGING_BYTES (32u << 20)

static __device__ __align__(256) unsigned char g_rtvla_static_staging[RTVLA_STATIC_STAGING_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
unsigned char *g_static_addr[kMaxDevices] = {};

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Device address of the staging array on device `dev` (which must be current).  The name
// g_rtvla_static_staging is only a host-side stand-in in host code; the address kernels and
// copies may use comes from cudaGetSymbolAddress, looked up once per device.
rtvla_status static_staging(int dev, unsigned char **out) {
  if (dev < 0 || dev >= kMaxDevices) return RTVLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_addr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_rtvla_static_staging);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return RTVLA_ERR_CUDA;
    }
    g_static_addr[dev] = static_cast<unsigned char *>(p);
  }
  *out = g_static_addr[dev];
  return RTVLA_OK;
}
}  // namespace

extern "C" rtvla_status rtvla_sample_actions_host_static(rtvla_ctx *c, const float *noise, const void *kv_k,
                                                         const void *kv_v, const int32_t *valid_len, int batch,
                                                         int prefix_cap, float *actions_out, void *stream) {
  if (!c || !noise || !kv_k || !kv_v || !valid_len || !actions_out) return RTVLA_ERR_INVALID_ARG;
  if (c->variant != RTVLA_VARIANT_PI05) return RTVLA_ERR_INVALID_ARG;  // π0 needs the state
  if (batch < 1 || prefix_cap < 1) return RTVLA_ERR_INVALID_ARG;
  if (batch > c->Bmax || prefix_cap > c->Pmax) return RTVLA_ERR_SHAPE;
  if (c->engine == RTVLA_ENGINE_PERSISTENT && !use_persistent(c, batch)) return RTVLA_ERR_UNSUPPORTED;
  const size_t kv_elems = (size_t)c->L * batch * prefix_cap * HD;
  const size_t io = (size_t)batch * c->Ca * A;
  const size_t off_act = round256(io * 4);
  const size_t off_vl = off_act + round256(io * 4);
  const size_t off_k = off_vl + round256((size_t)batch * 4);
  const size_t off_v = off_k + round256(kv_elems * 2);
  const size_t total = off_v + round256(kv_elems * 2);
  if (total > RTVLA_STATIC_STAGING_BYTES) return RTVLA_ERR_SHAPE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (dev != c->device) return RTVLA_ERR_INVALID_ARG;
  unsigned char *base = nullptr;
  rtvla_status s = static_staging(dev, &base);
  if (s != RTVLA_OK) return s;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float *d_noise = reinterpret_cast<float *>(base);
  float *d_act = reinterpret_cast<float *>(base + off_act);
  int *d_vl = reinterpret_cast<int *>(base + off_vl);
  bf16 *d_k = reinterpret_cast<bf16 *>(base + off_k);
  bf16 *d_v = reinterpret_cast<bf16 *>(base + off_v);
  const cudaMemcpyKind hd = cudaMemcpyHostToDevice;
  if (cudaMemcpyAsync(d_noise, noise, io * 4, hd, st) != cudaSuccess ||
      cudaMemcpyAsync(d_k, kv_k, kv_elems * 2, hd, st) != cudaSuccess ||
      cudaMemcpyAsync(d_v, kv_v, kv_elems * 2, hd, st) != cudaSuccess ||
      cudaMemcpyAsync(d_vl, valid_len, (size_t)batch * 4, hd, st) != cudaSuccess)
    return RTVLA_ERR_CUDA;
  CallArgs a;
  std::memset(&a, 0, sizeof(a));
  a.noise = d_noise;
  a.actions = d_act;
  a.kv_k = d_k;
  a.kv_v = d_v;
  a.valid_len = d_vl;
  a.batch = batch;
  a.cap = prefix_cap;
  if (cudaMemcpyAsync(c->args_dn, &a, sizeof(a), hd, st) != cudaSuccess) return RTVLA_ERR_CUDA;
  // The engine rtvla_sample_actions would pick: the persistent kernel (one launch, nothing
  // allocated: its per-call tensor maps are encoded on the host); else a graph already
  // captured for this shape is replayed; otherwise the same kernels are launched directly,
  // so that this call never instantiates anything.
  auto it = c->graphs_dn.find(std::make_pair(batch, prefix_cap));
  if (use_persistent(c, batch)) {
    rtvla_kv kv;
    kv.k = d_k;
    kv.v = d_v;
    kv.valid_len = d_vl;
    kv.batch = batch;
    kv.prefix_cap = prefix_cap;
    if (launch_persistent(c, c->args_dn, &kv, st) != cudaSuccess) {
      cudaGetLastError();
      return RTVLA_ERR_CUDA;
    }
  } else if (it != c->graphs_dn.end()) {
    if (cudaGraphLaunch(it->second.exec, st) != cudaSuccess) return RTVLA_ERR_CUDA;
  } else {
    int n = 0;
    if (enqueue_denoise(c, c->args_dn, batch, prefix_cap, st, nullptr, c->S - 1, &n) != cudaSuccess)
      return RTVLA_ERR_CUDA;
  }
  if (cudaMemcpyAsync(actions_out, d_act, io * 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return RTVLA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return RTVLA_ERR_CUDA;
  return RTVLA_OK;
}
