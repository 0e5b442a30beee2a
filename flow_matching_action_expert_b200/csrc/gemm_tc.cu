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
// epilogue: TMEM -> registers (x gate) -> a [TN tokens][128 features] fp32 tile in the freed
// pipeline stages -> one TMA bulk reduce-add (split K or accumulate) or bulk store per 64
// tokens.  Every wait is bounded (DevCtl::timeout_ns).
#include "common.cuh"
#include "kernels.h"

namespace rtvla {

template <int TN>
struct GemmCfg {
  static constexpr int W_BYTES = 128 * 128;  // 128 rows x 64 bf16
  static constexpr int X_BYTES = TN * 128;   // TN rows x 64 bf16
  static constexpr int STAGE = W_BYTES + X_BYTES;
  static constexpr int STAGES = (TN <= 64) ? 8 : (TN <= 128 ? 6 : 4);
  static constexpr int TMEM_COLS = TN <= 32 ? 32 : (TN <= 64 ? 64 : (TN <= 128 ? 128 : 256));
  static constexpr int SMEM = STAGES * STAGE + 1024 + 256;
};

template <int TN>
__global__ void __launch_bounds__(192, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
              const __grid_constant__ CUtensorMap tmO, GemmParams p) {
  using G = GemmCfg<TN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + G::STAGES * G::STAGE);
  uint64_t *empty = full + G::STAGES;
  uint64_t *done = empty + G::STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // token tiles vary fastest, so the CTAs that share a weight tile run together and all but
  // the first find it in L2
  const int m0 = blockIdx.x * TN;
  const int n0 = blockIdx.y * 128;
  const int kb_total = p.K >> 6;
  const int kb0 = blockIdx.z * p.kb_per_split;
  const int nkb = min(p.kb_per_split, kb_total - kb0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < G::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
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
    if (lane == 0 && nkb > 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      for (int i = 0; i < nkb; ++i) {
        const int s = i % G::STAGES;
        const uint32_t ph = (i / G::STAGES) & 1;
        if (i >= G::STAGES && !mbar_wait(&empty[s], ph ^ 1, p.ctl, 101)) break;
        uint8_t *st = smem + s * G::STAGE;
        mbar_arrive_expect_tx(&full[s], G::STAGE);
        tma_load_2d(st, &tmW, &full[s], (kb0 + i) * 64, p.w_row0 + n0, pol_w);
        tma_load_2d(st + G::W_BYTES, &tmX, &full[s], (kb0 + i) * 64, m0, pol_x);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, TN);
      for (int i = 0; i < nkb; ++i) {
        const int s = i % G::STAGES;
        const uint32_t ph = (i / G::STAGES) & 1;
        if (!mbar_wait(&full[s], ph, p.ctl, 102)) break;
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * G::STAGE);
        const uint32_t b = a + G::W_BYTES;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tmem, sdesc_k128(a + 32 * k), sdesc_k128(b + 32 * k), idesc, (i > 0 || k > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      umma_commit(done);
    }
  } else if (nkb > 0) {
    // epilogue: warp (2..5) & 3 selects the TMEM lane quadrant it may access; the tile reuses
    // the pipeline stages (every TMA load into them has been consumed once `done` fires)
    static_assert(TN * 128 * 4 <= G::STAGES * G::STAGE, "epilogue tile fits the stages");
    float *tile = reinterpret_cast<float *>(smem);
    const int q = warp & 3;
    const int nl = q * 32 + lane;
    if (mbar_wait(done, 0, p.ctl, 103)) {
      tc_fence_after();
      const float sc = p.col_scale ? p.col_scale[n0 + nl] : 1.0f;
#pragma unroll 1
      for (int c = 0; c < TN; c += 32) {
        float v[32];
        if (m0 + c < p.M) {
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c, v);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) tile[(c + j) * 128 + nl] = (m0 + c + j < p.M) ? v[j] * sc : 0.f;
      }
    }
    fence_proxy_async_shared();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (warp == 2 && lane == 0) {
      for (int t = 0; t < TN && m0 + t < p.M; t += 64) {
        if (p.atomic)
          tma_reduce_add_2d(&tmO, tile + t * 128, n0, m0 + t);
        else
          tma_store_2d(&tmO, tile + t * 128, n0, m0 + t);
      }
      bulk_commit();
      bulk_wait_read0();  // the tile must stay valid until the bulk copies have read it
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, G::TMEM_COLS);
  }
}

template <int TN>
static cudaError_t launch_tn(const CUtensorMap &tmW, const CUtensorMap &tmX, const CUtensorMap &tmO,
                             const GemmParams &p, int n_tiles, int m_tiles, int splits, cudaStream_t st) {
  using G = GemmCfg<TN>;
  dim3 grid(m_tiles, n_tiles, splits);
  k_gemm_tc<TN><<<grid, 192, G::SMEM, st>>>(tmW, tmX, tmO, p);
  return cudaGetLastError();
}

cudaError_t gemm_init_attributes() {
  cudaError_t e = cudaFuncSetAttribute(k_gemm_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg<64>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_gemm_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg<128>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_gemm_tc<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg<256>::SMEM);
  return e;
}

// Chooses the token tile and the K split so that about one wave of 148 SMs is busy.
GemmPlan gemm_plan(int M, int N, int K, int sm_count) {
  GemmPlan g;
  // a 128 x 256 x 16 MMA costs about as much as 128 x 128 x 16 (and 128 x 64 x 16) on sm_100a,
  // so past 128 rows the widest token tile wins even with its padding
  g.tn = (M <= 64) ? 64 : (M <= 128 ? 128 : 256);
  g.m_tiles = (M + g.tn - 1) / g.tn;
  g.n_tiles = N / 128;
  const int kb_total = K / 64;
  const int units = g.n_tiles * g.m_tiles;
  int splits = (sm_count + units - 1) / units;
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
  GemmParams p;
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
  const CUtensorMap &tmX = xm.m[gemm_tile_index(g.tn)];
  switch (g.tn) {
    case 64: return launch_tn<64>(tmW, tmX, tmO, p, g.n_tiles, g.m_tiles, g.splits, st);
    case 128: return launch_tn<128>(tmW, tmX, tmO, p, g.n_tiles, g.m_tiles, g.splits, st);
    default: return launch_tn<256>(tmW, tmX, tmO, p, g.n_tiles, g.m_tiles, g.splits, st);
  }
}

}  // namespace rtvla
