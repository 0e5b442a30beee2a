// Row-wise kernels of the denoise step and the prefix pass.
//
// Sources (Realtime-VLA tech blog): "Per-layer processing (PiGemmaDecoderLayer.forward)"
// for the op order, kernel list entries "adarms_norm_style_proj" (RMS statistics, (1 +
// scale) * x_norm + shift, gate kept apart), "matmul_rope_qkv" (RoPE applied to the QKV
// output, three destinations Q/K/V) and "Scalar ops in GEMM epilogues" (token statistics
// computed first, the normalisation factor applied after the GEMM accumulation).
//
// The AdaRMS of the expert is split accordingly: this file produces bf16(h * (1 + scale))
// and r = rsqrt(mean(h^2) + eps); the GEMM consumer multiplies its accumulator by r and
// adds shift @ W^T, a per-(step, layer) bias tabulated at create time.
#include "common.cuh"
#include "kernels.h"

namespace rtvla {

namespace {
__device__ __forceinline__ float block_sum_256(float v, float *red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = (l < 8) ? red[l] : 0.f;
  return warp_sum(s);
}
}  // namespace

// x = noise (copy through the call's argument block).  The expert runs Ct token rows per
// sample; the first `first` of them (the π0 state token) carry no action and get x = 0.
__global__ void k_init_x(const CallArgs *ca, float *x, int n, int Ct, int first) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int m = i >> 5, a = i & 31, b = m / Ct, j = m % Ct;
  x[i] = j < first ? 0.f : ca->noise[((size_t)b * (Ct - first) + (j - first)) * 32 + a];
}

// π0 suffix rows of one step ("Running VLAs at Real-time Speed" summary, "How": the two
// linears of the action time encoder folded, the step's time rows tabulated before SiLU).
// Row m of sample b = m / Ct: the state token (j = 0): h = W_s state_b + b_s and a zero GEMM
// operand; an action token: operand bf16(SiLU(W_fold x + c_k)) and h = b_out of the
// action-time MLP, to which the following GEMM adds operand @ W_out^T.
__global__ void __launch_bounds__(256) k_pi0_in(const float *x, const float *w_fold, const float *c_k,
                                                 const bf16 *w_st, const float *b_st, const float *b_ato,
                                                 const CallArgs *ca, float *h, bf16 *op, int Ct) {
  __shared__ float xs[32];
  const int m = blockIdx.x, b = m / Ct, j = m % Ct;
  if (threadIdx.x < 32) xs[threadIdx.x] = j == 0 ? ca->state[b * 32 + threadIdx.x] : x[m * 32 + threadIdx.x];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int n = threadIdx.x + 256 * k;
    if (j == 0) {
      const uint4 *wr = reinterpret_cast<const uint4 *>(w_st + n * 32);
      float acc = b_st[n];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = wr[q];
        const bf16 *e = reinterpret_cast<const bf16 *>(&v);
#pragma unroll
        for (int t = 0; t < 8; ++t) acc += bf2f(e[t]) * xs[q * 8 + t];
      }
      h[(size_t)m * 1024 + n] = acc;
      op[(size_t)m * 1024 + n] = f2bf(0.f);
    } else {
      const float4 *wr = reinterpret_cast<const float4 *>(w_fold + n * 32);
      float acc = c_k[n];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 v = wr[q];
        acc += v.x * xs[4 * q] + v.y * xs[4 * q + 1] + v.z * xs[4 * q + 2] + v.w * xs[4 * q + 3];
      }
      op[(size_t)m * 1024 + n] = f2bf(acc / (1.0f + __expf(-acc)));
      h[(size_t)m * 1024 + n] = b_ato[n];
    }
  }
}

// h[m][:] = x[m][:] @ W_in^T + b_in   (action_in_proj, 32 -> 1024)
__global__ void __launch_bounds__(256) k_action_in(const float *x, const bf16 *w_in, const float *b_in, float *h) {
  __shared__ float xs[32];
  const int m = blockIdx.x;
  if (threadIdx.x < 32) xs[threadIdx.x] = x[m * 32 + threadIdx.x];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int n = threadIdx.x + 256 * k;
    const uint4 *wr = reinterpret_cast<const uint4 *>(w_in + n * 32);
    float acc = b_in[n];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 v = wr[q];
      const bf16 *e = reinterpret_cast<const bf16 *>(&v);
#pragma unroll
      for (int j = 0; j < 8; ++j) acc += bf2f(e[j]) * xs[q * 8 + j];
    }
    h[(size_t)m * 1024 + n] = acc;
  }
}

// op = bf16(h * (1 + scale)), r = rsqrt(mean(h^2) + eps)   (width 1024)
__global__ void __launch_bounds__(256) k_adanorm(const float *h, const float *s1p, bf16 *op, float *r, float eps) {
  __shared__ float red[8];
  const int m = blockIdx.x;
  const float4 v = reinterpret_cast<const float4 *>(h + (size_t)m * 1024)[threadIdx.x];
  const float ss = block_sum_256(v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w, red);
  const float4 s = reinterpret_cast<const float4 *>(s1p)[threadIdx.x];
  uint2 o;
  o.x = pack_bf16(v.x * s.x, v.y * s.y);
  o.y = pack_bf16(v.z * s.z, v.w * s.w);
  reinterpret_cast<uint2 *>(op + (size_t)m * 1024)[threadIdx.x] = o;
  if (threadIdx.x == 0) r[m] = rsqrtf(ss * (1.0f / 1024.0f) + eps);
}

// QKV epilogue: y = r * acc + bias; RoPE (pairs d, d+128) at position Lv_b + j on the 8 query
// heads and the key; Q -> [M][2048], K_s, V_s -> [M][256] (bf16).  Clears acc.  Thread t owns
// 4 consecutive d of the rotated pairs in one head (288 pair groups: 8 query heads + the key,
// 32 per head) and, for t < 64, 4 consecutive columns of V; every load is issued before any
// store.
__global__ void __launch_bounds__(256) k_qkv_post(float *__restrict__ acc, const float *__restrict__ r,
                                                  const float *__restrict__ bias, const CallArgs *ca, int C,
                                                  const float *__restrict__ rc, const float *__restrict__ rs,
                                                  int rope_rows, bf16 *__restrict__ q, bf16 *__restrict__ ks,
                                                  bf16 *__restrict__ vs, DevCtl *ctl) {
  const int m = blockIdx.x;
  const int b = m / C, j = m % C;
  int pos = ca->valid_len[b] + j;
  if (pos < 0 || pos >= rope_rows) {
    if (threadIdx.x == 0) set_error(ctl, DEVERR_BOUNDS, 301);
    pos = pos < 0 ? 0 : rope_rows - 1;
  }
  float *a = acc + (size_t)m * 2560;
  const float rr = r[m];
  // two pair groups per thread (the first 32 threads take a third), loaded together
  float4 x1[2], x2[2], b1[2], b2[2], co[2], si[2];
  int grp[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    grp[k] = threadIdx.x + k * 256;
    const int g = grp[k] < 288 ? grp[k] : 0;
    const int head = g >> 5, d = (g & 31) * 4;
    const int c1 = head * 256 + d;
    x1[k] = *reinterpret_cast<const float4 *>(a + c1);
    x2[k] = *reinterpret_cast<const float4 *>(a + c1 + 128);
    b1[k] = *reinterpret_cast<const float4 *>(bias + c1);
    b2[k] = *reinterpret_cast<const float4 *>(bias + c1 + 128);
    co[k] = *reinterpret_cast<const float4 *>(rc + (size_t)pos * 128 + d);
    si[k] = *reinterpret_cast<const float4 *>(rs + (size_t)pos * 128 + d);
  }
  float4 vx = make_float4(0, 0, 0, 0), vb = vx;
  if (threadIdx.x < 64) {
    vx = *reinterpret_cast<const float4 *>(a + 2304 + threadIdx.x * 4);
    vb = *reinterpret_cast<const float4 *>(bias + 2304 + threadIdx.x * 4);
  }
  __syncthreads();  // every read of this row's accumulator is done before it is cleared
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    if (grp[k] >= 288) continue;
    const int head = grp[k] >> 5, d = (grp[k] & 31) * 4;
    const float *u = reinterpret_cast<const float *>(&x1[k]), *w = reinterpret_cast<const float *>(&x2[k]);
    const float *bu = reinterpret_cast<const float *>(&b1[k]), *bw = reinterpret_cast<const float *>(&b2[k]);
    const float *cs = reinterpret_cast<const float *>(&co[k]), *sn = reinterpret_cast<const float *>(&si[k]);
    float y1[4], y2[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float p1 = rr * u[e] + bu[e], p2 = rr * w[e] + bw[e];
      y1[e] = p1 * cs[e] - p2 * sn[e];
      y2[e] = p2 * cs[e] + p1 * sn[e];
    }
    bf16 *dst = head < 8 ? q + (size_t)m * 2048 + head * 256 : ks + (size_t)m * 256;
    uint2 lo, hi;
    lo.x = pack_bf16(y1[0], y1[1]);
    lo.y = pack_bf16(y1[2], y1[3]);
    hi.x = pack_bf16(y2[0], y2[1]);
    hi.y = pack_bf16(y2[2], y2[3]);
    *reinterpret_cast<uint2 *>(dst + d) = lo;
    *reinterpret_cast<uint2 *>(dst + d + 128) = hi;
  }
  if (threadIdx.x < 64) {
    uint2 o;
    o.x = pack_bf16(rr * vx.x + vb.x, rr * vx.y + vb.y);
    o.y = pack_bf16(rr * vx.z + vb.z, rr * vx.w + vb.w);
    *reinterpret_cast<uint2 *>(vs + (size_t)m * 256 + threadIdx.x * 4) = o;
  }
  for (int i = threadIdx.x; i < 2560 / 4; i += 256) reinterpret_cast<float4 *>(a)[i] = make_float4(0, 0, 0, 0);
}

// out[m][j] = bf16(GELU_tanh(r*g + bg) * (r*u + bu)), g = acc[m][j], u = acc[m][F + j].  Clears acc.
// Every load of a thread (F / 1024 groups of 4 columns) is issued before any store.
__global__ void __launch_bounds__(256) k_gelu_mul(float *__restrict__ acc, const float *__restrict__ r,
                                                  const float *__restrict__ bias, bf16 *__restrict__ out, int F) {
  const int m = blockIdx.x;
  float *a = acc + (size_t)m * 2 * F;
  const float rr = r ? r[m] : 1.0f;
  const int ng = F / 1024;
#pragma unroll 1
  for (int g0 = 0; g0 < ng; g0 += 4) {
    float4 g[4], u[4], bg[4], bu[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j = (g0 + k) * 1024 + threadIdx.x * 4;
      if (g0 + k < ng) {
        g[k] = *reinterpret_cast<const float4 *>(a + j);
        u[k] = *reinterpret_cast<const float4 *>(a + F + j);
        bg[k] = bias ? *reinterpret_cast<const float4 *>(bias + j) : make_float4(0, 0, 0, 0);
        bu[k] = bias ? *reinterpret_cast<const float4 *>(bias + F + j) : make_float4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (g0 + k >= ng) break;
      const int j = (g0 + k) * 1024 + threadIdx.x * 4;
      uint2 o;
      o.x = pack_bf16(gelu_tanh(rr * g[k].x + bg[k].x) * (rr * u[k].x + bu[k].x),
                      gelu_tanh(rr * g[k].y + bg[k].y) * (rr * u[k].y + bu[k].y));
      o.y = pack_bf16(gelu_tanh(rr * g[k].z + bg[k].z) * (rr * u[k].z + bu[k].z),
                      gelu_tanh(rr * g[k].w + bg[k].w) * (rr * u[k].w + bu[k].w));
      *reinterpret_cast<uint2 *>(out + (size_t)m * F + j) = o;
      *reinterpret_cast<float4 *>(a + j) = make_float4(0, 0, 0, 0);
      *reinterpret_cast<float4 *>(a + F + j) = make_float4(0, 0, 0, 0);
    }
  }
}

// Final AdaRMS (scale, shift) + action_out_proj with dt folded in + Euler:
// x[m] += n @ (dt W_out)^T + dt b_out.  Writes the actions when asked.
__global__ void __launch_bounds__(256) k_final(const float *h, const float *s1p, const float *shift, const float *w_out,
                                               const float *b_out, float *x, int final_norm, float eps,
                                               const CallArgs *ca, int write_actions, int Ct, int first) {
  __shared__ float n[1024];
  __shared__ float red[8];
  const int m = blockIdx.x;
  if (m % Ct < first) return;  // the π0 state token: no action
  const size_t arow = (size_t)(m / Ct) * (Ct - first) + (m % Ct - first);
  const float4 v = reinterpret_cast<const float4 *>(h + (size_t)m * 1024)[threadIdx.x];
  const float ss = block_sum_256(v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w, red);
  float4 y = v;
  if (final_norm) {
    const float r = rsqrtf(ss * (1.0f / 1024.0f) + eps);
    const float4 s = reinterpret_cast<const float4 *>(s1p)[threadIdx.x];
    const float4 t = reinterpret_cast<const float4 *>(shift)[threadIdx.x];
    y = make_float4(r * v.x * s.x + t.x, r * v.y * s.y + t.y, r * v.z * s.z + t.z, r * v.w * s.w + t.w);
  }
  reinterpret_cast<float4 *>(n)[threadIdx.x] = y;
  __syncthreads();
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int a = w * 4 + k;
    const float *wr = w_out + a * 1024;
    float acc = 0.f;
    for (int d = l; d < 1024; d += 32) acc += n[d] * wr[d];
    acc = warp_sum(acc);
    if (l == 0) {
      const float nx = x[m * 32 + a] + acc + b_out[a];
      x[m * 32 + a] = nx;
      if (write_actions) ca->actions[arow * 32 + a] = nx;
    }
  }
}

// ---------------------------------------------------------------------------------------
// prefix pass

// valid_len[b] = number of 1s in the pad mask; flags a mask whose valid tokens are not first.
__global__ void k_pf_mask(const CallArgs *ca, int P, DevCtl *ctl) {
  const int b = blockIdx.x;
  const uint8_t *mk = ca->mask + (size_t)b * P;
  int cnt = 0, bad = 0;
  for (int j = threadIdx.x; j < P; j += blockDim.x) {
    const int v = mk[j] != 0;
    cnt += v;
    if (v && j > 0 && mk[j - 1] == 0) bad = 1;
  }
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  bad = __reduce_or_sync(0xffffffffu, bad);
  __shared__ int sc[32], sb[32];
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    sc[w] = cnt;
    sb[w] = bad;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int c = 0, bb = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
      c += sc[i];
      bb |= sb[i];
    }
    ca->valid_out[b] = c;
    if (bb) set_error(ctl, DEVERR_MASK, 401);
  }
}

// x (fp32 residual) = embeddings
__global__ void k_pf_embed(const CallArgs *ca, float *x, size_t n) {
  const size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (i >= n) return;
  const uint4 v = *reinterpret_cast<const uint4 *>(ca->embeds + i);
  const bf16 *e = reinterpret_cast<const bf16 *>(&v);
  float4 *o = reinterpret_cast<float4 *>(x + i);
  o[0] = make_float4(bf2f(e[0]), bf2f(e[1]), bf2f(e[2]), bf2f(e[3]));
  o[1] = make_float4(bf2f(e[4]), bf2f(e[5]), bf2f(e[6]), bf2f(e[7]));
}

// op = bf16(x * rsqrt(mean(x^2) + eps)); the RMSNorm weight (1 + w) is folded into the next GEMM.
__global__ void __launch_bounds__(256) k_rmsnorm(const float *x, bf16 *op, int Dp, float eps) {
  __shared__ float red[8];
  const int m = blockIdx.x;
  const float *xr = x + (size_t)m * Dp;
  float ss = 0.f;
  for (int i = threadIdx.x * 4; i < Dp; i += 1024) {
    const float4 v = *reinterpret_cast<const float4 *>(xr + i);
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = block_sum_256(ss, red);
  const float r = rsqrtf(ss / (float)Dp + eps);
  for (int i = threadIdx.x * 4; i < Dp; i += 1024) {
    const float4 v = *reinterpret_cast<const float4 *>(xr + i);
    uint2 o;
    o.x = pack_bf16(v.x * r, v.y * r);
    o.y = pack_bf16(v.z * r, v.w * r);
    *reinterpret_cast<uint2 *>(op + (size_t)m * Dp + i) = o;
  }
}

// Prefill QKV epilogue: RoPE at position j (the valid tokens come first, so cumsum(mask) - 1
// = j on them); Q -> q, K and V -> the output cache of this layer.  Clears acc.
__global__ void __launch_bounds__(256) k_pf_qkv_post(float *acc, const CallArgs *ca, int layer, int P,
                                                     const float *rc, const float *rs, int rope_rows, bf16 *q,
                                                     DevCtl *ctl) {
  const int m = blockIdx.x;
  const int b = m / P, j = m % P;
  int pos = j;
  if (pos >= rope_rows) {
    if (threadIdx.x == 0) set_error(ctl, DEVERR_BOUNDS, 302);
    pos = rope_rows - 1;
  }
  float *a = acc + (size_t)m * 2560;
  const size_t kvo = (((size_t)layer * ca->batch + b) * ca->cap + j) * 256;
  const float *cr = rc + (size_t)pos * 128;
  const float *sr = rs + (size_t)pos * 128;
  for (int i = threadIdx.x; i < 9 * 128; i += 256) {
    const int head = i >> 7, d = i & 127;
    const int c1 = head * 256 + d, c2 = c1 + 128;
    const float x1 = a[c1], x2 = a[c2];
    const float co = cr[d], si = sr[d];
    const float y1 = x1 * co - x2 * si, y2 = x2 * co + x1 * si;
    if (head < 8) {
      q[(size_t)m * 2048 + c1] = f2bf(y1);
      q[(size_t)m * 2048 + c2] = f2bf(y2);
    } else {
      ca->kvo_k[kvo + d] = f2bf(y1);
      ca->kvo_k[kvo + d + 128] = f2bf(y2);
    }
  }
  for (int d = threadIdx.x; d < 256; d += 256) ca->kvo_v[kvo + d] = f2bf(a[2304 + d]);
  __syncthreads();
  for (int i = threadIdx.x; i < 2560 / 4; i += 256) reinterpret_cast<float4 *>(a)[i] = make_float4(0, 0, 0, 0);
}

// ---------------------------------------------------------------------------------------
// create-time precompute in fp64

// out[s][r] = sum_k W[r][k] * vecs[s][k] + bias[r]  (one warp per row r, S <= 64)
__global__ void k_rows_dot_f64(const bf16 *W, int R, int Kd, const double *vecs, int S, const bf16 *bias,
                               double *out) {
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int l = threadIdx.x & 31;
  if (r >= R) return;
  const bf16 *wr = W + (size_t)r * Kd;
  for (int s = 0; s < S; ++s) {
    const double *v = vecs + (size_t)s * Kd;
    double acc = 0.0;
    for (int k = l; k < Kd; k += 32) acc += (double)bf2f(wr[k]) * v[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (l == 0) out[(size_t)s * R + r] = acc + (bias ? (double)bf2f(bias[r]) : 0.0);
  }
}

// out[r][k] = bf16(W[r][k] * (1 + gamma[k]))  (Gemma RMSNorm weight folded into the next Linear)
__global__ void k_fold_cols(const bf16 *W, int R, int Kd, const bf16 *gamma, bf16 *out) {
  const size_t n = (size_t)R * Kd;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int k = (int)(i % Kd);
    out[i] = f2bf(bf2f(W[i]) * (1.0f + bf2f(gamma[k])));
  }
}

__global__ void k_scale_to_f32(const bf16 *w, int n, double s, float *out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = (float)((double)bf2f(w[i]) * s);
}

// ---------------------------------------------------------------------------------------
// launchers
cudaError_t launch_init_x(const CallArgs *ca, float *x, int n, int Ct, int first, cudaStream_t st) {
  k_init_x<<<(n + 255) / 256, 256, 0, st>>>(ca, x, n, Ct, first);
  return cudaGetLastError();
}
cudaError_t launch_pi0_in(const float *x, const float *w_fold, const float *c_k, const bf16 *w_st, const float *b_st,
                          const float *b_ato, const CallArgs *ca, float *h, bf16 *op, int M, int Ct, cudaStream_t st) {
  k_pi0_in<<<M, 256, 0, st>>>(x, w_fold, c_k, w_st, b_st, b_ato, ca, h, op, Ct);
  return cudaGetLastError();
}
cudaError_t launch_action_in(const float *x, const bf16 *w_in, const float *b_in, float *h, int M, cudaStream_t st) {
  k_action_in<<<M, 256, 0, st>>>(x, w_in, b_in, h);
  return cudaGetLastError();
}
cudaError_t launch_adanorm(const float *h, const float *s1p, bf16 *op, float *r, int M, float eps, cudaStream_t st) {
  k_adanorm<<<M, 256, 0, st>>>(h, s1p, op, r, eps);
  return cudaGetLastError();
}
cudaError_t launch_qkv_post(float *acc, const float *r, const float *bias, const CallArgs *ca, int C,
                            const float *rope_cos, const float *rope_sin, int rope_rows, bf16 *q, bf16 *ks,
                            bf16 *vs, int M, DevCtl *ctl, cudaStream_t st) {
  k_qkv_post<<<M, 256, 0, st>>>(acc, r, bias, ca, C, rope_cos, rope_sin, rope_rows, q, ks, vs, ctl);
  return cudaGetLastError();
}
cudaError_t launch_gelu_mul(float *acc, const float *r, const float *bias, bf16 *out, int M, int F, cudaStream_t st) {
  k_gelu_mul<<<M, 256, 0, st>>>(acc, r, bias, out, F);
  return cudaGetLastError();
}
cudaError_t launch_final(const float *h, const float *s1p, const float *shift, const float *w_out, const float *b_out,
                         float *x, int M, int final_norm, float eps, const CallArgs *ca, int write_actions,
                         int Ct, int first, cudaStream_t st) {
  k_final<<<M, 256, 0, st>>>(h, s1p, shift, w_out, b_out, x, final_norm, eps, ca, write_actions, Ct, first);
  return cudaGetLastError();
}
cudaError_t launch_pf_mask(const CallArgs *ca, int B, int P, DevCtl *ctl, cudaStream_t st) {
  k_pf_mask<<<B, 256, 0, st>>>(ca, P, ctl);
  return cudaGetLastError();
}
cudaError_t launch_pf_embed(const CallArgs *ca, float *x, int M, int Dp, cudaStream_t st) {
  const size_t n = (size_t)M * Dp;
  k_pf_embed<<<(unsigned)((n / 8 + 255) / 256), 256, 0, st>>>(ca, x, n);
  return cudaGetLastError();
}
cudaError_t launch_rmsnorm(const float *x, bf16 *op, int M, int Dp, float eps, cudaStream_t st) {
  k_rmsnorm<<<M, 256, 0, st>>>(x, op, Dp, eps);
  return cudaGetLastError();
}
cudaError_t launch_pf_qkv_post(float *acc, const CallArgs *ca, int layer, int P, const float *rope_cos,
                               const float *rope_sin, int rope_rows, bf16 *q, int M, DevCtl *ctl, cudaStream_t st) {
  k_pf_qkv_post<<<M, 256, 0, st>>>(acc, ca, layer, P, rope_cos, rope_sin, rope_rows, q, ctl);
  return cudaGetLastError();
}
cudaError_t launch_rows_dot_f64(const bf16 *W, int R, int Kd, const double *vecs, int S, const bf16 *bias,
                                double *out, cudaStream_t st) {
  k_rows_dot_f64<<<(R + 7) / 8, 256, 0, st>>>(W, R, Kd, vecs, S, bias, out);
  return cudaGetLastError();
}
cudaError_t launch_fold_cols(const bf16 *W, int R, int Kd, const bf16 *gamma, bf16 *out, cudaStream_t st) {
  k_fold_cols<<<1184, 256, 0, st>>>(W, R, Kd, gamma, out);
  return cudaGetLastError();
}
cudaError_t launch_scale_to_f32(const bf16 *w, int n, double s, float *out, cudaStream_t st) {
  k_scale_to_f32<<<(n + 255) / 256, 256, 0, st>>>(w, n, s, out);
  return cudaGetLastError();
}

}  // namespace rtvla

namespace rtvla {

// One CTA per guarded buffer: both bands are compared with the fill byte 16 bytes at a time;
// a band that changed is reported (DEVERR_GUARD, where = 700 + buffer index) and refilled.
__global__ void k_check_guards(const GuardRegion *regions, DevCtl *ctl) {
  const GuardRegion r = regions[blockIdx.x];
  const uint4 fill4 = make_uint4(0xA5A5A5A5u, 0xA5A5A5A5u, 0xA5A5A5A5u, 0xA5A5A5A5u);
  static_assert(GUARD_FILL == 0xA5, "fill word");
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  uint4 *bands[2] = {reinterpret_cast<uint4 *>(r.base),
                     reinterpret_cast<uint4 *>(r.base + GUARD_BYTES + r.bytes)};
  for (int b = 0; b < 2; ++b)
    for (int i = threadIdx.x; i < GUARD_BYTES / 16; i += blockDim.x) {
      const uint4 v = bands[b][i];
      if (v.x != fill4.x || v.y != fill4.y || v.z != fill4.z || v.w != fill4.w) {
        bad = 1;
        bands[b][i] = fill4;
      }
    }
  __syncthreads();
  if (threadIdx.x == 0 && bad) set_error(ctl, DEVERR_GUARD, 700 + (int)blockIdx.x);
}

cudaError_t launch_check_guards(const GuardRegion *regions, int n, DevCtl *ctl, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  k_check_guards<<<n, 256, 0, st>>>(regions, ctl);
  return cudaGetLastError();
}

}  // namespace rtvla
