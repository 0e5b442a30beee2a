// Multi-query attention over [valid prefix keys ; suffix keys] (Realtime-VLA tech blog,
// kernel list "softmax_kernel_prefix_suffix": the prefix KV cache joined with the decoder's
// own K/V, the prefix valid length read at run time).  The padding mask is a length: key j
// of sample b is prefix token j for j < Lv_b and suffix token j - Lv_b after it, so padded
// prefix slots are never loaded.
//
// One CTA = one sample, 16 queries, all 8 query heads (warp w = head w; they share the one
// KV head), one contiguous split of the keys.  K/V chunks of 64 keys are staged in shared
// memory once and read by all 8 warps; S = Q K^T and O = P V run on mma.sync tensor-core
// tiles with an online (flash) softmax in fp32.  Several splits are merged by a second
// kernel with log-sum-exp weights.  Calls with at least 64 (sample, query block) units run the
// tcgen05 kernel of attention_tc.cu instead (attn_launch decides); both write the same
// partials, so k_attn_combine serves either.
#include "common.cuh"
#include "kernels.h"

namespace rtvla {

namespace {
constexpr int HD = 256;
constexpr int NH = 8;
constexpr int KC = 64;     // keys per chunk
constexpr int QB = 16;     // queries per CTA
constexpr int LDS = HD + 8;  // padded shared row (528 bytes) -> conflict-free ldmatrix
constexpr int SMEM_ATTN = (NH * QB + 2 * KC) * LDS * 2;
}  // namespace

__global__ void __launch_bounds__(256, 1) k_attn(AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  bf16 *Qs = reinterpret_cast<bf16 *>(smem_raw);  // [NH][QB][LDS]
  bf16 *Ks = Qs + NH * QB * LDS;                  // [KC][LDS]
  bf16 *Vs = Ks + KC * LDS;                       // [KC][LDS]

  const int split = blockIdx.x, qb = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const CallArgs *ca = p.ca;
  const int B = ca->batch, cap = ca->cap;
  int lv = ca->valid_len[b];
  if (lv < 0 || lv > cap) {
    if (threadIdx.x == 0 && split == 0 && qb == 0) set_error(p.ctl, DEVERR_BOUNDS, 201);
    lv = lv < 0 ? 0 : cap;
  }
  const size_t lay = (size_t)p.layer * B * cap * HD + (size_t)b * cap * HD;
  const bf16 *kpre = ca->kv_k + lay;
  const bf16 *vpre = ca->kv_v + lay;
  const int total = lv + p.n_suf;
  const int k_begin = split * p.keys_per_split;
  const int k_end = min(total, k_begin + p.keys_per_split);

  // stage the 16 x 8 query rows: all of a thread's loads in flight before its stores
  {
    constexpr int NQL = NH * QB * (HD / 8) / 256;
    uint4 qv[NQL];
#pragma unroll
    for (int i = 0; i < NQL; ++i) {
      const int idx = threadIdx.x + i * 256;
      const int c8 = idx % (HD / 8), row = (idx / (HD / 8)) % QB, h = idx / (QB * (HD / 8));
      const int qi = qb * QB + row;
      qv[i] = qi < p.nq ? *reinterpret_cast<const uint4 *>(p.q + (size_t)(b * p.nq + qi) * p.q_ld + h * HD + c8 * 8)
                        : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < NQL; ++i) {
      const int idx = threadIdx.x + i * 256;
      const int c8 = idx % (HD / 8), row = (idx / (HD / 8)) % QB, h = idx / (QB * (HD / 8));
      *reinterpret_cast<uint4 *>(Qs + (h * QB + row) * LDS + c8 * 8) = qv[i];
    }
  }

  float o[32][4];
#pragma unroll
  for (int i = 0; i < 32; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int g = lane >> 2, t = lane & 3;
  const bf16 *Qw = Qs + warp * QB * LDS;

#pragma unroll 1
  for (int c0 = k_begin; c0 < k_end; c0 += KC) {
    // this chunk's K / V rows: every load of the thread in flight before any store (the
    // prefix rows come from HBM; one round trip instead of eight)
    constexpr int NKL = KC * (HD / 8) / 256;
    uint4 kv[NKL], vv[NKL];
#pragma unroll
    for (int i = 0; i < NKL; ++i) {
      const int idx = threadIdx.x + i * 256;
      const int c8 = idx % (HD / 8), j = c0 + idx / (HD / 8);
      kv[i] = vv[i] = make_uint4(0, 0, 0, 0);
      if (j < lv) {
        kv[i] = *reinterpret_cast<const uint4 *>(kpre + (size_t)j * HD + c8 * 8);
        vv[i] = *reinterpret_cast<const uint4 *>(vpre + (size_t)j * HD + c8 * 8);
      } else if (j < k_end) {
        const size_t off = ((size_t)b * p.n_suf + (j - lv)) * HD + c8 * 8;
        kv[i] = *reinterpret_cast<const uint4 *>(p.ksuf + off);
        vv[i] = *reinterpret_cast<const uint4 *>(p.vsuf + off);
      }
    }
    __syncthreads();  // previous chunk fully consumed (and Q staged on the first pass)
#pragma unroll
    for (int i = 0; i < NKL; ++i) {
      const int idx = threadIdx.x + i * 256;
      const int c8 = idx % (HD / 8), r = idx / (HD / 8);
      *reinterpret_cast<uint4 *>(Ks + r * LDS + c8 * 8) = kv[i];
      *reinterpret_cast<uint4 *>(Vs + r * LDS + c8 * 8) = vv[i];
    }
    __syncthreads();

    // S = Q K^T for 16 queries x 64 keys
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(a0, a1, a2, a3, smem_u32(Qw + (lane & 15) * LDS + kk * 16 + (lane >> 4) * 8));
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        uint32_t b0, b1, b2, b3;
        const int r = nt * 8 + (lane & 7) + ((lane >> 4) << 3);
        const int c = kk * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4(b0, b1, b2, b3, smem_u32(Ks + r * LDS + c));
        mma_16816(s[nt], a0, a1, a2, a3, b0, b1);
        mma_16816(s[nt + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    // mask, scale, online softmax (rows g and g + 8 of this warp's tile)
    float cm0 = -INFINITY, cm1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = c0 + nt * 8 + 2 * t + (e & 1);
        const float v = (key < k_end) ? s[nt][e] * p.scale_log2 : -INFINITY;
        s[nt][e] = v;
        if (e < 2) cm0 = fmaxf(cm0, v); else cm1 = fmaxf(cm1, v);
      }
    }
    cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, 1));
    cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, 2));
    cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, 1));
    cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, 2));
    const float nm0 = fmaxf(m0, cm0), nm1 = fmaxf(m1, cm1);
    const float r0 = (nm0 == -INFINITY) ? 0.f : nm0;
    const float r1 = (nm1 == -INFINITY) ? 0.f : nm1;
    const float al0 = exp2f(m0 - r0), al1 = exp2f(m1 - r1);
    m0 = nm0;
    m1 = nm1;
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = exp2f(s[nt][0] - r0);
      s[nt][1] = exp2f(s[nt][1] - r0);
      s[nt][2] = exp2f(s[nt][2] - r1);
      s[nt][3] = exp2f(s[nt][3] - r1);
      ps0 += s[nt][0] + s[nt][1];
      ps1 += s[nt][2] + s[nt][3];
    }
    l0 = l0 * al0 + ps0;
    l1 = l1 * al1 + ps1;
#pragma unroll
    for (int dt = 0; dt < 32; ++dt) {
      o[dt][0] *= al0;
      o[dt][1] *= al0;
      o[dt][2] *= al1;
      o[dt][3] *= al1;
    }
    // O += P V
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
      const uint32_t a0 = pack_bf16(s[2 * kt][0], s[2 * kt][1]);
      const uint32_t a1 = pack_bf16(s[2 * kt][2], s[2 * kt][3]);
      const uint32_t a2 = pack_bf16(s[2 * kt + 1][0], s[2 * kt + 1][1]);
      const uint32_t a3 = pack_bf16(s[2 * kt + 1][2], s[2 * kt + 1][3]);
#pragma unroll
      for (int dt = 0; dt < 32; dt += 2) {
        uint32_t b0, b1, b2, b3;
        const int r = kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = dt * 8 + (lane >> 4) * 8;
        ldsm_x4_t(b0, b1, b2, b3, smem_u32(Vs + r * LDS + c));
        mma_16816(o[dt], a0, a1, a2, a3, b0, b1);
        mma_16816(o[dt + 1], a0, a1, a2, a3, b2, b3);
      }
    }
  }

  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

  const int qa = qb * QB + g, qc = qa + 8;
  if (p.n_splits == 1) {
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
    for (int dt = 0; dt < 32; ++dt) {
      const int d = warp * HD + dt * 8 + 2 * t;
      if (qa < p.nq)
        *reinterpret_cast<uint32_t *>(p.out + (size_t)(b * p.nq + qa) * (NH * HD) + d) =
            pack_bf16(o[dt][0] * i0, o[dt][1] * i0);
      if (qc < p.nq)
        *reinterpret_cast<uint32_t *>(p.out + (size_t)(b * p.nq + qc) * (NH * HD) + d) =
            pack_bf16(o[dt][2] * i1, o[dt][3] * i1);
    }
  } else {
    const size_t base = ((size_t)b * p.n_splits + split) * p.nq;
#pragma unroll
    for (int dt = 0; dt < 32; ++dt) {
      const int d = dt * 8 + 2 * t;
      if (qa < p.nq)
        *reinterpret_cast<float2 *>(p.opart + ((base + qa) * NH + warp) * HD + d) = make_float2(o[dt][0], o[dt][1]);
      if (qc < p.nq)
        *reinterpret_cast<float2 *>(p.opart + ((base + qc) * NH + warp) * HD + d) = make_float2(o[dt][2], o[dt][3]);
    }
    if (t == 0) {
      if (qa < p.nq) *reinterpret_cast<float2 *>(p.mlpart + ((base + qa) * NH + warp) * 2) = make_float2(m0, l0);
      if (qc < p.nq) *reinterpret_cast<float2 *>(p.mlpart + ((base + qc) * NH + warp) * 2) = make_float2(m1, l1);
    }
  }
}

// Merges the splits of one query row: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
__global__ void __launch_bounds__(256) k_attn_combine(AttnParams p) {
  const int row = blockIdx.x;  // b * nq + i
  const int b = row / p.nq, i = row % p.nq;
  const int h = threadIdx.x >> 5, d0 = (threadIdx.x & 31) * 8;
  float M = -INFINITY;
#pragma unroll 4
  for (int s = 0; s < p.n_splits; ++s)
    M = fmaxf(M, p.mlpart[((((size_t)b * p.n_splits + s) * p.nq + i) * NH + h) * 2]);
  const float ref = (M == -INFINITY) ? 0.f : M;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float L = 0.f;
#pragma unroll 4
  for (int s = 0; s < p.n_splits; ++s) {
    const size_t r = (((size_t)b * p.n_splits + s) * p.nq + i) * NH + h;
    const float2 ml = *reinterpret_cast<const float2 *>(p.mlpart + r * 2);
    const float w = exp2f(ml.x - ref);
    L += w * ml.y;
    const float4 *src = reinterpret_cast<const float4 *>(p.opart + r * HD + d0);
    const float4 x0 = src[0], x1 = src[1];
    acc[0] += w * x0.x; acc[1] += w * x0.y; acc[2] += w * x0.z; acc[3] += w * x0.w;
    acc[4] += w * x1.x; acc[5] += w * x1.y; acc[6] += w * x1.z; acc[7] += w * x1.w;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint4 v;
  v.x = pack_bf16(acc[0] * inv, acc[1] * inv);
  v.y = pack_bf16(acc[2] * inv, acc[3] * inv);
  v.z = pack_bf16(acc[4] * inv, acc[5] * inv);
  v.w = pack_bf16(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4 *>(p.out + (size_t)row * (NH * HD) + h * HD + d0) = v;
}

int attn_splits(int batch, int nq, int max_keys, int sm_count, int *keys_per_split) {
  const int qblocks = (nq + QB - 1) / QB;
  const int chunks = (max_keys + KC - 1) / KC;
  const int base = batch * qblocks;
  // as many splits as keep every CTA in one wave over the SMs
  int splits = sm_count / base;
  if (splits > chunks) splits = chunks;
  if (splits < 1) splits = 1;
  const int cps = (chunks + splits - 1) / splits;
  *keys_per_split = cps * KC;
  return (chunks + cps - 1) / cps;
}

cudaError_t attn_init_attributes() {
  const cudaError_t e = cudaFuncSetAttribute(k_attn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ATTN);
  return e != cudaSuccess ? e : attn_tc_init_attributes();
}

int attn_keys(int prefix_cap, int n_suf) { return KC * ((prefix_cap + KC - 1) / KC + (n_suf + KC - 1) / KC); }

cudaError_t attn_launch(const AttnParams &p, int batch, cudaStream_t st) {
  // The tcgen05 kernel pays once there are enough (sample, query block) units to fill the
  // GPU; below that its fixed costs lose to this kernel.  Measured on B200: 3-view batch 64
  // 63.2 -> 55.3 ms, batch 16 24.0 -> 22.6 ms; batch 4 equal; batch 1 and the 544-token
  // prefill 3-7% slower.
  const int qblocks = (p.nq + QB - 1) / QB;
  cudaError_t e;
  if (batch * qblocks >= 64) {
    e = attn_tc_launch(p, batch, st);
  } else {
    dim3 grid(p.n_splits, qblocks, batch);
    k_attn<<<grid, 256, SMEM_ATTN, st>>>(p);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess || p.n_splits == 1) return e;
  k_attn_combine<<<batch * p.nq, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace rtvla
