// Skinny bf16 GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// out[m][n] (+)= s[n] * sum_k X[m][k] * W[n][k]      (fp32 accumulation in TMEM)
//
// The weight is the A operand (M = 128 output features per tile) and the activation is the
// B operand (N = TN tokens), so a 63-token chunk fills one N = 64 tile and the weight
// stream — the part that is HBM-bound at batch 1 — is split over many CTAs along N and K.
// Split-K partial sums are added with fp32 reductions into an output that is either zero
// (scratch, cleared by its consumer) or the fp32 residual stream itself (gated residual
// "res + (x @ W) * gate" of the Realtime-VLA tech blog, kernel list "matmul_small_res_gate").
//
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer and TMEM owner, warps 2..5 =
// epilogue: TMEM -> registers (x gate) -> a [64 tokens][128 features] fp32 box in shared
// memory -> one TMA bulk reduce-add (split K or accumulate) or bulk store per 64 tokens.
// Gated-GELU form (GemmParams::glu, the tech blog's "Gated Linear Layer融合 (§4.2)"): a tile's
// 128 weight rows are 64 gate rows and the 64 matching up rows, and the epilogue turns the
// box into bf16 GELU_tanh(r*g + b_g) * (r*u + b_u) for 64 features, stored by one TMA copy.
// Every wait is bounded (DevCtl::timeout_ns).
#include "common.cuh"
#include "kernels.h"

namespace rtvla {

// DEEP (token tiles of 256 only): a 4-stage ring and one epilogue box instead of 3 stages and
// two boxes.  It pays where a CTA has several tiles or long K slices, so that the ring, not
// the epilogue, sets the pace: measured on B200, +9-11% on the 544-token prefill's gate/up
// and down GEMMs, -12% on its one-round QKV GEMM.
template <int TN, bool DEEP = false>
struct GemmCfg {
  static constexpr int W_BYTES = 128 * 128;  // 128 rows x 64 bf16
  static constexpr int X_BYTES = TN * 128;   // TN rows x 64 bf16
  static constexpr int STAGE = W_BYTES + X_BYTES;
  static constexpr int STAGES = (TN <= 64) ? 6 : (TN <= 128 ? 5 : (DEEP ? 4 : 3));
  static constexpr int BOXES = DEEP ? 1 : 2;  // fp32 epilogue boxes
  static constexpr int EPI = 64 * 128 * 4;   // one 64-token x 128-feature fp32 epilogue box
  static constexpr int TMEM_COLS = 2 * (TN <= 32 ? 32 : TN);  // two accumulators
  static constexpr int SMEM = STAGES * STAGE + BOXES * EPI + 1024 + 256;
  static_assert(SMEM <= 232448, "shared memory per CTA");
};

// Tile t of the launch: token tile t % m_tiles, weight tile (t / m_tiles) % n_tiles, K split
// t / (m_tiles * n_tiles).  Token tiles vary fastest so the CTAs that share a weight tile run
// together and all but the first find it in L2.
struct TileIdx {
  int m0, n0, kb0, nkb;
};
template <int TN>
__device__ __forceinline__ TileIdx tile_at(const GemmParams &p, int t) {
  TileIdx r;
  const int mi = t % p.m_tiles, rest = t / p.m_tiles;
  r.m0 = mi * TN;
  r.n0 = (rest % p.n_tiles) * 128;
  r.kb0 = (rest / p.n_tiles) * p.kb_per_split;
  r.nkb = min(p.kb_per_split, (p.K >> 6) - r.kb0);
  return r;
}

// Persistent: CTA c computes tiles c, c + grid, ...  Warp roles: warp 0 = TMA producer
// through a STAGES-deep ring, warp 1 = MMA issuer alternating between two TMEM accumulators,
// warps 2..5 = epilogue, which drains one accumulator (64 tokens at a time through two
// shared-memory boxes and TMA bulk reduce / store) while the MMA fills the other.
template <int TN, bool DEEP = false>
__global__ void __launch_bounds__(192, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
              const __grid_constant__ CUtensorMap tmO, GemmParams p) {
  using G = GemmCfg<TN, DEEP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *epi = reinterpret_cast<float *>(smem + G::STAGES * G::STAGE);  // [2][64][128]
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + G::STAGES * G::STAGE + G::BOXES * G::EPI);
  uint64_t *empty = full + G::STAGES;
  uint64_t *acc_full = empty + G::STAGES;  // [2]
  uint64_t *acc_empty = acc_full + 2;      // [2]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.m_tiles * p.n_tiles * p.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < G::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, G::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const TileIdx ti = tile_at<TN>(p, t);
        for (int i = 0; i < ti.nkb; ++i, ++it) {
          const int s = it % G::STAGES;
          if (it >= (uint32_t)G::STAGES && !mbar_wait(&empty[s], ((it / G::STAGES) & 1) ^ 1, p.ctl, 101)) {
            ok = false;
            break;
          }
          uint8_t *st = smem + s * G::STAGE;
          mbar_arrive_expect_tx(&full[s], G::STAGE);
          if (p.glu) {
            // gate rows f0 .. f0 + 63 over A rows 0..63, the matching up rows over A rows 64..127
            const int f0 = ti.n0 >> 1;
            tma_load_2d(st, &tmW, &full[s], (ti.kb0 + i) * 64, p.w_row0 + f0, pol_w);
            tma_load_2d(st + G::W_BYTES / 2, &tmW, &full[s], (ti.kb0 + i) * 64, p.w_row0 + (p.N >> 1) + f0, pol_w);
          } else {
            tma_load_2d(st, &tmW, &full[s], (ti.kb0 + i) * 64, p.w_row0 + ti.n0, pol_w);
          }
          tma_load_2d(st + G::W_BYTES, &tmX, &full[s], (ti.kb0 + i) * 64, ti.m0, pol_x);
        }
      }
      // every issued copy must land before the CTA may exit
      const uint32_t first = it > (uint32_t)G::STAGES ? it - G::STAGES : 0;
      for (uint32_t j = first; j < it; ++j) mbar_wait(&full[j % G::STAGES], (j / G::STAGES) & 1, p.ctl, 104);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, TN);
      uint32_t it = 0;
      int local = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++local) {
        const TileIdx ti = tile_at<TN>(p, t);
        const int b = local & 1;
        // the epilogue must have drained this accumulator (used two tiles ago)
        if (local >= 2 && !mbar_wait(&acc_empty[b], ((local >> 1) & 1) ^ 1, p.ctl, 105)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * (G::TMEM_COLS / 2));
        for (int i = 0; i < ti.nkb; ++i, ++it) {
          const int s = it % G::STAGES;
          if (!mbar_wait(&full[s], (it / G::STAGES) & 1, p.ctl, 102)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(smem + s * G::STAGE);
          const uint32_t bx = a + G::W_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(d, sdesc_k128(a + 32 * k), sdesc_k128(bx + 32 * k), idesc, (i > 0 || k > 0) ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&acc_full[b]);
      }
    }
  } else {
    // epilogue: warp (2..5) & 3 selects the TMEM lane quadrant (features) it may access
    const int q = warp & 3;
    const int nl = q * 32 + lane;
    const bool leader = warp == 2 && lane == 0;
    int local = 0;
    uint32_t nbox = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++local) {
      const TileIdx ti = tile_at<TN>(p, t);
      const int b = local & 1;
      if (!mbar_wait(&acc_full[b], (local >> 1) & 1, p.ctl, 103)) break;
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(b * (G::TMEM_COLS / 2)) + ((uint32_t)(q * 32) << 16);
      const float sc = p.col_scale ? p.col_scale[ti.n0 + nl] : 1.0f;
      for (int c0 = 0; c0 < TN && ti.m0 + c0 < p.M; c0 += 64, ++nbox) {
        float *box = epi + (G::BOXES == 2 ? (nbox & 1) : 0) * (64 * 128);
        if (leader && nbox >= (uint32_t)G::BOXES) {  // the copy that last read this box is done
          if (G::BOXES == 2)
            bulk_wait_read<1>();
          else
            bulk_wait_read<0>();
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll 1
        for (int c = c0; c < c0 + 64 && c < TN; c += 32) {
          float v[32];
          if (ti.m0 + c < p.M) {
            tmem_ld32(d + (uint32_t)c, v);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.f;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) box[(c - c0 + j) * 128 + nl] = (ti.m0 + c + j < p.M) ? v[j] * sc : 0.f;
        }
        if (p.glu) {
          // box columns 0..63 hold the gate features, 64..127 the up features: thread t takes
          // feature t % 64 for 32 of the 64 tokens, then the bf16 results replace the box as
          // [64 tokens][64 features] with 128-byte swizzle, stored by one TMA copy
          asm volatile("bar.sync 1, 128;" ::: "memory");
          const int t = (warp - 2) * 32 + lane;
          const int f = t & 63, th = t >> 6;
          const int f0 = ti.n0 >> 1;
          const float bg = p.glu_bias ? p.glu_bias[f0 + f] : 0.f;
          const float bu = p.glu_bias ? p.glu_bias[(p.N >> 1) + f0 + f] : 0.f;
          float mv[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int tok = th * 32 + j, row = ti.m0 + c0 + tok;
            const float rr = (p.glu_r != nullptr && row < p.M) ? p.glu_r[row] : 1.f;
            mv[j] = gelu_tanh(rr * box[tok * 128 + f] + bg) * (rr * box[tok * 128 + 64 + f] + bu);
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");  // every read of the fp32 box is done
          bf16 *ob = reinterpret_cast<bf16 *>(box);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int tok = th * 32 + j;
            ob[tok * 64 + ((((f >> 3) ^ (tok & 7)) << 3) | (f & 7))] = f2bf(mv[j]);
          }
          fence_proxy_async_shared();
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (leader) {
            tma_store_2d(&tmO, box, f0, ti.m0 + c0);
            bulk_commit();
          }
        } else {
          fence_proxy_async_shared();
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (leader) {
            if (p.atomic)
              tma_reduce_add_2d(&tmO, box, ti.n0, ti.m0 + c0);
            else
              tma_store_2d(&tmO, box, ti.n0, ti.m0 + c0);
            bulk_commit();
          }
        }
      }
      // the accumulator has been read: hand it back to the MMA issuer
      tc_fence_before();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (leader) mbar_arrive(&acc_empty[b]);
    }
    if (leader) bulk_wait0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, G::TMEM_COLS);
  }
}

template <int TN, bool DEEP = false>
static cudaError_t launch_tn(const CUtensorMap &tmW, const CUtensorMap &tmX, const CUtensorMap &tmO,
                             const GemmParams &p, int sm_count, cudaStream_t st) {
  using G = GemmCfg<TN, DEEP>;
  const int tiles = p.m_tiles * p.n_tiles * p.splits;
  k_gemm_tc<TN, DEEP><<<dim3(tiles < sm_count ? tiles : sm_count), 192, G::SMEM, st>>>(tmW, tmX, tmO, p);
  return cudaGetLastError();
}

cudaError_t gemm_init_attributes() {
  cudaError_t e = cudaFuncSetAttribute(k_gemm_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg<64>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_gemm_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg<128>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_gemm_tc<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg<256>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_gemm_tc<256, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg<256, true>::SMEM);
  return e;
}

static cudaError_t launch_plan(const CUtensorMap &tmW, const XMaps &xm, const CUtensorMap &tmO, int tn,
                               const GemmParams &p, int sm_count, cudaStream_t st) {
  const CUtensorMap &tmX = xm.m[gemm_tile_index(tn)];
  switch (tn) {
    case 64: return launch_tn<64>(tmW, tmX, tmO, p, sm_count, st);
    case 128: return launch_tn<128>(tmW, tmX, tmO, p, sm_count, st);
    default:
      // several tiles per CTA, or a long K slice: the deeper ring
      if (p.m_tiles * p.n_tiles * p.splits > sm_count || p.kb_per_split >= 32)
        return launch_tn<256, true>(tmW, tmX, tmO, p, sm_count, st);
      return launch_tn<256>(tmW, tmX, tmO, p, sm_count, st);
  }
}

// Chooses the token tile and the K split (at most one round of tiles over the SMs).
GemmPlan gemm_plan(int M, int N, int K, int sm_count) {
  GemmPlan g;
  // a 128 x 256 x 16 MMA costs about as much as 128 x 128 x 16 (and 128 x 64 x 16) on sm_100a,
  // so past 128 rows the widest token tile wins even with its padding
  g.tn = (M <= 64) ? 64 : (M <= 128 ? 128 : 256);
  g.m_tiles = (M + g.tn - 1) / g.tn;
  g.n_tiles = N / 128;
  const int kb_total = K / 64;
  const int units = g.n_tiles * g.m_tiles;
  // split K only as far as one round of tiles fits the SMs: a second, partial round would cost
  // a whole tile time, and splits beyond that only add reduction traffic
  int splits = sm_count / units;
  if (splits < 1) splits = 1;
  if (splits > kb_total) splits = kb_total;
  g.kb_per_split = (kb_total + splits - 1) / splits;
  g.splits = (kb_total + g.kb_per_split - 1) / g.kb_per_split;
  return g;
}

int gemm_tile_index(int tn) { return tn <= 64 ? 0 : (tn <= 128 ? 1 : 2); }

cudaError_t gemm_launch(const CUtensorMap &tmW, int w_row0, const XMaps &xm, int M, int N, int K, float *out,
                        const CUtensorMap &tmO, int ldo, const float *col_scale, bool accumulate, DevCtl *ctl,
                        int sm_count, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  GemmPlan g = gemm_plan(M, N, K, sm_count);
  GemmParams p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.w_row0 = w_row0;
  p.kb_per_split = g.kb_per_split;
  p.out = out;
  p.ldo = ldo;
  p.col_scale = col_scale;
  p.atomic = (accumulate || g.splits > 1) ? 1 : 0;
  p.ctl = ctl;
  p.m_tiles = g.m_tiles;
  p.n_tiles = g.n_tiles;
  p.splits = g.splits;
  const int pairs = gemm2_clusters();
  if (g.tn == 256 && (g.n_tiles & 1) == 0 && pairs > 0) {
    // SM pairs: 256 weight rows x 256 tokens per pair tile; K split only as far as one round
    // of pair tiles fits the clusters
    const int kb_total = K / 64;
    const int units = g.m_tiles * (g.n_tiles >> 1);
    int splits = pairs / units;
    if (splits < 1) splits = 1;
    if (splits > kb_total) splits = kb_total;
    p.kb_per_split = (kb_total + splits - 1) / splits;
    p.splits = (kb_total + p.kb_per_split - 1) / p.kb_per_split;
    p.atomic = (accumulate || p.splits > 1) ? 1 : 0;
    return gemm2_launch(tmW, xm.m[1], tmO, p, st);
  }
  return launch_plan(tmW, xm, tmO, g.tn, p, sm_count, st);
}

bool gemm_glu_applies(int M, int F, int K, int sm_count) { return gemm_plan(M, 2 * F, K, sm_count).splits == 1; }

cudaError_t gemm_launch_glu(const CUtensorMap &tmW64, int w_row0, const XMaps &xm, int M, int F, int K,
                            const CUtensorMap &tmM, const float *r, const float *bias, DevCtl *ctl, int sm_count,
                            cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  const GemmPlan g = gemm_plan(M, 2 * F, K, sm_count);
  if (g.splits != 1) return cudaErrorInvalidValue;
  GemmParams p{};
  p.M = M;
  p.N = 2 * F;
  p.K = K;
  p.w_row0 = w_row0;
  p.kb_per_split = g.kb_per_split;
  p.ldo = F;
  p.ctl = ctl;
  p.m_tiles = g.m_tiles;
  p.n_tiles = g.n_tiles;
  p.splits = 1;
  p.glu = 1;
  p.glu_r = r;
  p.glu_bias = bias;
  return launch_plan(tmW64, xm, tmM, g.tn, p, sm_count, st);
}

}  // namespace rtvla
