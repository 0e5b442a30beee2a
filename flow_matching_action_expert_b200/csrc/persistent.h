// Persistent engine of the denoise loop (one cooperative kernel per call; batch 1, chunk <= 64).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace rtvla {

struct PersistParams {
  const CallArgs *ca;       // noise, actions, prefix cache, valid length
  unsigned int *bar;        // grid-barrier counter (zeroed by the per-call argument copy)
  int L, S, C;
  int final_norm;
  float eps;
  float scale_log2;         // log2(e) / sqrt(head_dim)
  int attn_splits, attn_cps;  // attention key splits and 32-key chunks per split
  int ca_cap;                 // token stride of this call's prefix cache
  // folded weights and per-(step, layer) tables (library-owned)
  const bf16 *w_in;
  const float *b_in, *w_out, *b_out;
  const float *s1p_attn, *gate_attn, *s1p_ffn, *gate_ffn, *bias_qkv, *bias_gu, *s1p_fin, *shift_fin;
  const float *rope_cos, *rope_sin;
  // activations (library-owned static buffers)
  float *x, *h, *acc_qkv, *acc_gu, *ss_attn, *ss_ffn, *opart, *mlpart;
  bf16 *o;                  // attention output [64][2048] (O-projection operand)
  bf16 *qb, *ks, *vs;       // finalised Q [64][2048], suffix K / V [64][256]
  DevCtl *ctl;
  // optional phase timestamps (globaltimer ns), [grid][max_phases][8]: 0 phase start,
  // 1 operand ready, 2 accumulator ready, 3 epilogue issued, 4 attention queries staged,
  // 5 first key chunk staged, 6 attention done, 7 barrier arrival; null unless the
  // environment variable RTVLA_PHASE_STAMPS names the file rtvla_destroy writes them to
  unsigned long long *stamps;
  int max_phases;
  // optional per-layer trace: at step trace_step the kernel writes h before layer 0 and after
  // every layer to trace, f32 [L + 1][C][1024]; null in normal calls
  float *trace;
  int trace_step;
  // π0 suffix (pi0 = 1): row 0 is the state token, rows 1 .. C-1 the action tokens; each
  // step's action tokens are W_ato SiLU(W_fold x + c_k) + b_ato, the state token W_st s + b_st
  int pi0;
  const float *w_fold, *c_tab, *b_ato, *b_st;  // fp32 [1024][32], [S][1024], [1024], [1024]
  const bf16 *w_ato, *w_st;                    // bf16 [1024][1024], [1024][32]
  bf16 *op_ato;                                // bf16 [64][1024]: SiLU(W_fold x + c_k) per row
};

int persistent_smem_bytes();
cudaError_t persistent_init_attributes();
bool persistent_fits(int sm_count);
void persistent_attn_plan(int cap, int chunk, int sm_count, int *splits, int *cps);
int persistent_max_splits(int sm_count);  // upper bound of the splits any plan returns
// Tensor maps of the persistent kernel.
struct PersistMaps {
  CUtensorMap w_qkv, w_o, w_gu, w_d;  // stacked bf16 weights, 64-column x 128-row boxes, 128B swizzle
  CUtensorMap r_qkv, r_gu, r_h;       // fp32 bulk-reduce targets acc_qkv, acc_gu, h (128 x 64 boxes)
  CUtensorMap l_h, l_gu;              // fp32 loads of h (4 x 8 KB tiles per box) and acc_gu (2 per box):
                                      // 3-D {32 cols, 64 rows, column blocks}, 128B swizzle per tile
  CUtensorMap l_o;                    // bf16 load of the attention output, 64 x 64 boxes, 128B swizzle
  CUtensorMap l_q;                    // bf16 finalised Q [64][2048], 64 x 64 boxes
  CUtensorMap l_kc, l_vc;             // this call's prefix cache [L * cap][256], 64 x 32 boxes (per call)
  CUtensorMap l_ks, l_vs;             // finalised suffix K / V [64][256], 64 x 32 boxes
};
cudaError_t persistent_launch(const PersistMaps &m, const PersistParams &p, int grid, cudaStream_t st);

}  // namespace rtvla
