// Image front-end kernels, sm_100a: the SigLIP-shaped vision tower and multi_modal_projector
// that turn each 224 x 224 camera view into 256 prefix embeddings (Realtime-VLA tech blog,
// "pi0.5 inference flow": encoder step 1 and the class hierarchy's vision_tower /
// multi_modal_projector).
//
// The dense contractions (patch embedding, QKV, O, fc1, fc2, projector) run on the tcgen05
// GEMM of gemm_tc.cu.  This file holds everything between them:
//   k_vis_embed  patch gather (the stride-14 convolution's operand, 588 values per patch padded
//                to 640) and the residual stream's start value (patch bias + position embedding)
//   k_vis_ln     LayerNorm of one token row to a bf16 GEMM operand; it also adds the bias of
//                the linear that the next GEMM accumulates into the residual stream, and sets
//                the next GEMM's own fp32 output rows to that GEMM's bias
//   k_vis_attn   multi-head attention inside one image (16 heads x 72 dims, 256 keys) on
//                mma.sync tensor-core tiles, one pass (all 256 keys fit)
//   k_vis_gelu   GELU_tanh of fc1's output (bias already in it) to bf16
//   k_vis_out    projector output x sqrt(2048) to bf16 rows of the caller's prefix buffer
#include "common.cuh"
#include "kernels.h"

namespace rtvla {

namespace {
constexpr int VW = VIS_WIDTH;      // 1152
constexpr int VT = VIS_TOKENS;     // 256 tokens per image
constexpr int VHD = 72;            // head dim
constexpr int VHDP = 80;           // head dim padded to whole 16-wide MMA k-steps
constexpr int VNH = 16;            // heads
constexpr int VIMG = 224, VPATCH = 14, VGRID = 16;
constexpr int VKP = VIS_PATCH_K;   // 640: 3 x 14 x 14 = 588 padded
constexpr int VKR = 588;
constexpr int VQKV = 3 * VW;       // 3456
constexpr int VOUT = VIS_OUT;      // 2048
constexpr int LDA = 88;            // shared row of 88 bf16 (176 bytes): conflict-free ldmatrix
constexpr int ATTN_SMEM = (2 * VT + 64) * LDA * 2;
static_assert(VHDP <= LDA, "padded head row");
}  // namespace

// ---------------------------------------------------------------------------------------
// patch gather + residual-stream start
//
// Blocks [0, nb_cols): one 16-byte group of 8 operand values per thread.  Row r = i * 256 + t
// (image i, patch t = py * 16 + px in raster order) holds pixel (c, 14 py + ky, 14 px + kx) at
// column c * 196 + ky * 14 + kx, the order of the convolution weight [out][c][ky][kx]; columns
// 588..639 are zero.  Blocks [nb_cols, ...): one float4 of h = table[t] per thread, the table
// being patch bias + position embedding (fp32, built at create).
__global__ void __launch_bounds__(256) k_vis_embed(const VisArgs *va, bf16 *cols, float *h, const float *table,
                                                   int n_img, int nb_cols) {
  if ((int)blockIdx.x < nb_cols) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= n_img * VT * (VKP / 8)) return;
    const int g8 = idx % (VKP / 8), r = idx / (VKP / 8);
    const int i = r / VT, t = r % VT, py = t / VGRID, px = t % VGRID;
    const float *img = va->images + (size_t)i * 3 * VIMG * VIMG;
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int k = g8 * 8 + e;
      float x = 0.f;
      if (k < VKR) {
        const int c = k / 196, rem = k - c * 196, ky = rem / VPATCH, kx = rem - ky * VPATCH;
        x = img[((size_t)c * VIMG + py * VPATCH + ky) * VIMG + px * VPATCH + kx];
      }
      v[e] = x;
    }
    uint4 o;
    o.x = pack_bf16(v[0], v[1]);
    o.y = pack_bf16(v[2], v[3]);
    o.z = pack_bf16(v[4], v[5]);
    o.w = pack_bf16(v[6], v[7]);
    *reinterpret_cast<uint4 *>(cols + (size_t)r * VKP + g8 * 8) = o;
  } else {
    const int idx = (blockIdx.x - nb_cols) * blockDim.x + threadIdx.x;
    if (idx >= n_img * VT * (VW / 4)) return;
    const int c4 = idx % (VW / 4), t = (idx / (VW / 4)) % VT;
    reinterpret_cast<float4 *>(h)[idx] = reinterpret_cast<const float4 *>(table)[(size_t)t * (VW / 4) + c4];
  }
}

// ---------------------------------------------------------------------------------------
// LayerNorm: one CTA of 288 threads per token row (1152 = 288 x 4)
//
// y = bf16((x - mean) / sqrt(var + eps) * gain + offset), biased variance, two-pass.  Then, in
// this order of effect: x += add (when add is given) and acc[row] := acc_init (when acc is
// given; acc_cols a multiple of 4).  The add is the bias of the linear whose output the next
// residual GEMM reduces into x; acc_init is the bias of the GEMM that reduces into acc.
__global__ void __launch_bounds__(288) k_vis_ln(float *x, const float *add, const float *gain, const float *offset,
                                                bf16 *y, float *acc, const float *acc_init, int acc_cols,
                                                float eps) {
  __shared__ float red[2][9];
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float4 *xr = reinterpret_cast<float4 *>(x + (size_t)row * VW);
  const float4 v = xr[tid];
  float s = warp_sum(v.x + v.y + v.z + v.w);
  if (lane == 0) red[0][warp] = s;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < 9; ++i) tot += red[0][i];
  const float mean = tot * (1.0f / VW);
  const float d0 = v.x - mean, d1 = v.y - mean, d2 = v.z - mean, d3 = v.w - mean;
  const float q = warp_sum(d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3);
  if (lane == 0) red[1][warp] = q;
  __syncthreads();
  float tq = 0.f;
#pragma unroll
  for (int i = 0; i < 9; ++i) tq += red[1][i];
  const float rstd = rsqrtf(tq * (1.0f / VW) + eps);
  const float4 g = reinterpret_cast<const float4 *>(gain)[tid];
  const float4 o = reinterpret_cast<const float4 *>(offset)[tid];
  *reinterpret_cast<uint2 *>(y + (size_t)row * VW + tid * 4) =
      make_uint2(pack_bf16(d0 * rstd * g.x + o.x, d1 * rstd * g.y + o.y),
                 pack_bf16(d2 * rstd * g.z + o.z, d3 * rstd * g.w + o.w));
  if (add) {
    const float4 a = reinterpret_cast<const float4 *>(add)[tid];
    xr[tid] = make_float4(v.x + a.x, v.y + a.y, v.z + a.z, v.w + a.w);
  }
  if (acc) {
    float4 *ar = reinterpret_cast<float4 *>(acc + (size_t)row * acc_cols);
    const float4 *ai = reinterpret_cast<const float4 *>(acc_init);
    for (int c = tid; c < acc_cols / 4; c += 288) ar[c] = ai[c];
  }
}

// ---------------------------------------------------------------------------------------
// attention inside one image: grid (256 / 64 query blocks, 16 heads, images), 4 warps; warp w
// takes queries qb * 64 + w * 16 .. + 15 of image blockIdx.z and head blockIdx.y.
//
// qkv: fp32 [rows][3456] = [q | k | v] with the biases in (head h at columns h * 72 of each
// third).  K, V (256 rows) and Q (64 rows) are staged as bf16 [row][88] with dims 72..79 zero;
// S = Q K^T for all 256 keys stays in registers (32 tiles of 8 keys), the softmax is exact
// (one max, one sum), and O = P V accumulates 10 tiles of 8 dims of which the first 9 are
// written: out bf16 [rows][1152], head h at columns h * 72.
__global__ void __launch_bounds__(128) k_vis_attn(const float *qkv, bf16 *out, float scale_log2) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  bf16 *Ks = reinterpret_cast<bf16 *>(smem_raw);  // [256][LDA]
  bf16 *Vs = Ks + VT * LDA;                         // [256][LDA]
  bf16 *Qs = Vs + VT * LDA;                         // [64][LDA]
  const int qb = blockIdx.x, h = blockIdx.y;
  const size_t row0 = (size_t)blockIdx.z * VT;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // staging: every load of a batch is issued before its stores (Q: one batch of 9 float4 per
  // thread; K and V: three batches of 12 + 12), so a CTA waits for 4 round trips, not 45
  const float *base = qkv + row0 * VQKV + h * VHD;
  {
    constexpr int QN = 64 * (VHD / 4) / 128;  // 9
    float4 qv[QN];
#pragma unroll
    for (int j = 0; j < QN; ++j) {
      const int idx = tid + j * 128, r = idx / (VHD / 4), c4 = idx % (VHD / 4);
      qv[j] = *reinterpret_cast<const float4 *>(base + (size_t)(qb * 64 + r) * VQKV + c4 * 4);
    }
#pragma unroll
    for (int j = 0; j < QN; ++j) {
      const int idx = tid + j * 128, r = idx / (VHD / 4), c4 = idx % (VHD / 4);
      *reinterpret_cast<uint2 *>(Qs + r * LDA + c4 * 4) =
          make_uint2(pack_bf16(qv[j].x, qv[j].y), pack_bf16(qv[j].z, qv[j].w));
    }
  }
  constexpr int KVN = VT * (VHD / 4) / 128;  // 36 float4 of K and 36 of V per thread
  constexpr int KB = 12;
  static_assert(KVN % KB == 0, "whole batches");
#pragma unroll 1
  for (int b0 = 0; b0 < KVN; b0 += KB) {
    float4 kv[KB], vv[KB];
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      const int idx = tid + (b0 + j) * 128, r = idx / (VHD / 4), c4 = idx % (VHD / 4);
      const float *src = base + (size_t)r * VQKV + c4 * 4;
      kv[j] = *reinterpret_cast<const float4 *>(src + VW);
      vv[j] = *reinterpret_cast<const float4 *>(src + 2 * VW);
    }
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      const int idx = tid + (b0 + j) * 128, r = idx / (VHD / 4), c4 = idx % (VHD / 4);
      *reinterpret_cast<uint2 *>(Ks + r * LDA + c4 * 4) =
          make_uint2(pack_bf16(kv[j].x, kv[j].y), pack_bf16(kv[j].z, kv[j].w));
      *reinterpret_cast<uint2 *>(Vs + r * LDA + c4 * 4) =
          make_uint2(pack_bf16(vv[j].x, vv[j].y), pack_bf16(vv[j].z, vv[j].w));
    }
  }
  for (int r = tid; r < VT; r += 128) {
    *reinterpret_cast<uint4 *>(Ks + r * LDA + VHD) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4 *>(Vs + r * LDA + VHD) = make_uint4(0, 0, 0, 0);
    if (r < 64) *reinterpret_cast<uint4 *>(Qs + r * LDA + VHD) = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();

  // S = Q K^T: 16 queries x 256 keys
  const bf16 *Qw = Qs + warp * 16 * LDA;
  float s[32][4];
#pragma unroll
  for (int i = 0; i < 32; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < VHDP / 16; ++kk) {
    uint32_t a0, a1, a2, a3;
    ldsm_x4(a0, a1, a2, a3, smem_u32(Qw + (lane & 15) * LDA + kk * 16 + (lane >> 4) * 8));
#pragma unroll
    for (int nt = 0; nt < 32; nt += 2) {
      uint32_t b0, b1, b2, b3;
      const int r = nt * 8 + (lane & 7) + ((lane >> 4) << 3);
      const int c = kk * 16 + ((lane >> 3) & 1) * 8;
      ldsm_x4(b0, b1, b2, b3, smem_u32(Ks + r * LDA + c));
      mma_16816(s[nt], a0, a1, a2, a3, b0, b1);
      mma_16816(s[nt + 1], a0, a1, a2, a3, b2, b3);
    }
  }
  // softmax over the 256 keys of rows g and g + 8 (a row is spread over the 4 lanes of a quad)
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 32; ++nt) {
    m0 = fmaxf(m0, fmaxf(s[nt][0], s[nt][1]));
    m1 = fmaxf(m1, fmaxf(s[nt][2], s[nt][3]));
  }
  m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
  m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
  m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
  m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
  float l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int nt = 0; nt < 32; ++nt) {
    s[nt][0] = exp2f((s[nt][0] - m0) * scale_log2);
    s[nt][1] = exp2f((s[nt][1] - m0) * scale_log2);
    s[nt][2] = exp2f((s[nt][2] - m1) * scale_log2);
    s[nt][3] = exp2f((s[nt][3] - m1) * scale_log2);
    l0 += s[nt][0] + s[nt][1];
    l1 += s[nt][2] + s[nt][3];
  }
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

  // O = P V: P's accumulator tiles 2kt, 2kt + 1 are the A operand of key step kt
  float o[VHDP / 8][4];
#pragma unroll
  for (int i = 0; i < VHDP / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
#pragma unroll
  for (int kt = 0; kt < VT / 16; ++kt) {
    const uint32_t a0 = pack_bf16(s[2 * kt][0], s[2 * kt][1]);
    const uint32_t a1 = pack_bf16(s[2 * kt][2], s[2 * kt][3]);
    const uint32_t a2 = pack_bf16(s[2 * kt + 1][0], s[2 * kt + 1][1]);
    const uint32_t a3 = pack_bf16(s[2 * kt + 1][2], s[2 * kt + 1][3]);
#pragma unroll
    for (int dt = 0; dt < VHDP / 8; dt += 2) {
      uint32_t b0, b1, b2, b3;
      const int r = kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int c = dt * 8 + (lane >> 4) * 8;
      ldsm_x4_t(b0, b1, b2, b3, smem_u32(Vs + r * LDA + c));
      mma_16816(o[dt], a0, a1, a2, a3, b0, b1);
      mma_16816(o[dt + 1], a0, a1, a2, a3, b2, b3);
    }
  }
  const float i0 = 1.f / l0, i1 = 1.f / l1;
  const int g = lane >> 2, t4 = lane & 3;
  const size_t qa = row0 + qb * 64 + warp * 16 + g, qc = qa + 8;
#pragma unroll
  for (int dt = 0; dt < VHD / 8; ++dt) {
    const int d = h * VHD + dt * 8 + 2 * t4;
    *reinterpret_cast<uint32_t *>(out + qa * VW + d) = pack_bf16(o[dt][0] * i0, o[dt][1] * i0);
    *reinterpret_cast<uint32_t *>(out + qc * VW + d) = pack_bf16(o[dt][2] * i1, o[dt][3] * i1);
  }
}

// ---------------------------------------------------------------------------------------
// out = bf16(GELU_tanh(acc)), 4 values per thread
__global__ void __launch_bounds__(256) k_vis_gelu(const float *acc, bf16 *out, int n4) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 v = reinterpret_cast<const float4 *>(acc)[i];
  reinterpret_cast<uint2 *>(out)[i] = make_uint2(pack_bf16(gelu_tanh(v.x), gelu_tanh(v.y)),
                                                 pack_bf16(gelu_tanh(v.z), gelu_tanh(v.w)));
}

// ---------------------------------------------------------------------------------------
// row r = i * 256 + j of acc [rows][2048] -> prefix row (b, v * 256 + j) of va->out
// [batch][ld][2048], b = i / views, v = i % views; 4 values per thread
__global__ void __launch_bounds__(256) k_vis_out(const VisArgs *va, const float *acc, int n_img, float scale) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_img * VT * (VOUT / 4)) return;
  const int c4 = idx % (VOUT / 4), r = idx / (VOUT / 4);
  const int i = r / VT, j = r % VT;
  const int views = va->views;
  const int b = i / views, v = i % views;
  const float4 x = reinterpret_cast<const float4 *>(acc)[idx];
  bf16 *dst = va->out + ((size_t)b * va->ld + (size_t)v * VT + j) * VOUT + c4 * 4;
  *reinterpret_cast<uint2 *>(dst) =
      make_uint2(pack_bf16(x.x * scale, x.y * scale), pack_bf16(x.z * scale, x.w * scale));
}

// ---------------------------------------------------------------------------------------
// launchers

cudaError_t vis_init_attributes() {
  return cudaFuncSetAttribute(k_vis_attn, cudaFuncAttributeMaxDynamicSharedMemorySize, ATTN_SMEM);
}

cudaError_t launch_vis_embed(const VisArgs *va, bf16 *cols, float *h, const float *table, int n_img,
                             cudaStream_t st) {
  const int nb_cols = (n_img * VT * (VKP / 8) + 255) / 256;
  const int nb_h = (n_img * VT * (VW / 4) + 255) / 256;
  k_vis_embed<<<nb_cols + nb_h, 256, 0, st>>>(va, cols, h, table, n_img, nb_cols);
  return cudaGetLastError();
}

cudaError_t launch_vis_ln(float *x, const float *add, const float *gain, const float *offset, bf16 *y, float *acc,
                          const float *acc_init, int acc_cols, int M, float eps, cudaStream_t st) {
  if ((acc && (acc_cols % 4 != 0 || !acc_init)) || M <= 0) return cudaErrorInvalidValue;
  k_vis_ln<<<M, 288, 0, st>>>(x, add, gain, offset, y, acc, acc_init, acc_cols, eps);
  return cudaGetLastError();
}

cudaError_t launch_vis_attn(const float *qkv, bf16 *out, int n_img, cudaStream_t st) {
  const float scale_log2 = (float)(1.4426950408889634 / 8.48528137423857);  // log2(e) / sqrt(72)
  k_vis_attn<<<dim3(VT / 64, VNH, n_img), 128, ATTN_SMEM, st>>>(qkv, out, scale_log2);
  return cudaGetLastError();
}

cudaError_t launch_vis_gelu(const float *acc, bf16 *out, int M, int cols, cudaStream_t st) {
  if (cols % 4 != 0) return cudaErrorInvalidValue;
  const int n4 = M * cols / 4;
  k_vis_gelu<<<(n4 + 255) / 256, 256, 0, st>>>(acc, out, n4);
  return cudaGetLastError();
}

cudaError_t launch_vis_out(const VisArgs *va, const float *acc, int n_img, cudaStream_t st) {
  const int n = n_img * VT * (VOUT / 4);
  k_vis_out<<<(n + 255) / 256, 256, 0, st>>>(va, acc, n_img, 45.254833995939045f);  // sqrt(2048)
  return cudaGetLastError();
}

}  // namespace rtvla
