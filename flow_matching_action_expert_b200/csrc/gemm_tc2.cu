// Skinny bf16 GEMM on an SM pair: the 2-CTA form of k_gemm_tc for token tiles of 256.
//
// out[m][n] (+)= s[n] * sum_k X[m][k] * W[n][k]      (fp32 accumulation in TMEM)
//
// A cluster of two CTAs computes one 256-weight-row x 256-token tile with tcgen05.mma
// .cta_group::2 (M = 256): CTA rank r holds weight rows n0 + 128 r .. + 127 (its half of A) and
// tokens m0 + 128 r .. + 127 (its half of B) in its own shared memory, and its TMEM receives
// the accumulator of its 128 weight rows for all 256 tokens.  Against two independent
// 128 x 256 tiles this halves the activation bytes each SM stages per MMA, so a deeper ring
// fits the same shared memory.
//
// Roles per CTA: warp 0 = TMA producer of this CTA's halves; warp 1 = the MMA issuer in CTA 0
// (in CTA 1 it relays "stage full" to CTA 0); warps 2..5 = epilogue of this CTA's rows.
// Every copy completes on its own CTA's barrier; CTA 1 forwards each completed stage to CTA 0
// with a remote mbarrier arrive, and CTA 0 commits each consumed stage back to both CTAs.
// Every wait is bounded (DevCtl::timeout_ns).
//
// The form is opt-in (RTVLA_PAIR_GEMM=1 at rtvla_create): on B200 it measured about half the
// rate of k_gemm_tc on the prefill and batch-64 shapes.
#include <cstdlib>

#include "common.cuh"
#include "kernels.h"

namespace rtvla {
namespace g2 {

constexpr int A_BYTES = 128 * 128;  // this CTA's 128 weight rows x 64 bf16
constexpr int B_BYTES = 128 * 128;  // this CTA's 128 tokens x 64 bf16
constexpr int STAGE = A_BYTES + B_BYTES;
constexpr int STAGES = 5;
constexpr int EPI = 64 * 128 * 4;   // one 64-token x 128-feature fp32 epilogue box
constexpr int TMEM_COLS = 512;      // two accumulators of 256 columns
constexpr int NBAR = 3 * STAGES + 5;
constexpr int SMEM = STAGES * STAGE + 2 * EPI + 1024 + NBAR * 8 + 16;
static_assert(SMEM <= 232448, "shared memory per CTA");

__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_ctas() {
  uint32_t n;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
  return n;
}
// shared::cluster address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t cluster_addr(const void *p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  return a;
}
__device__ __forceinline__ void remote_arrive(uint32_t caddr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ bool try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait with cluster-scope acquire (the barrier may be completed from the peer CTA)
__device__ __forceinline__ bool wait_c(uint64_t *bar, uint32_t parity, DevCtl *ctl, int where,
                                       uint64_t min_ns = 0) {
  const uint32_t a = smem_u32(bar);
#pragma unroll 1
  for (int i = 0; i < 64; ++i)
    if (try_wait_cluster(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  const uint64_t lim = ctl->timeout_ns > min_ns ? ctl->timeout_ns : min_ns;
#pragma unroll 1
  while (true) {
    if (try_wait_cluster(a, parity)) return true;
    if (globaltimer() - t0 > lim) {
      set_error(ctl, DEVERR_TIMEOUT, where);
      return false;
    }
  }
}
__device__ __forceinline__ void umma2_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrives on the barrier at cluster address `caddr` once every earlier pair MMA of this
// thread has completed
__device__ __forceinline__ void commit2(uint32_t caddr) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(caddr)
               : "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t *slot, uint32_t ncols) {  // whole warp, both CTAs
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Pair tile t: token tile t % m_tiles (256 tokens), weight pair tile (t / m_tiles) % (n_tiles / 2)
// (256 rows), K split t / (m_tiles * n_tiles / 2).
struct Tile2 {
  int m0, n0, kb0, nkb;
};
__device__ __forceinline__ Tile2 tile2_at(const GemmParams &p, int t) {
  Tile2 r;
  const int np = p.n_tiles >> 1;
  const int mi = t % p.m_tiles, rest = t / p.m_tiles;
  r.m0 = mi * 256;
  r.n0 = (rest % np) * 256;
  r.kb0 = (rest / np) * p.kb_per_split;
  r.nkb = min(p.kb_per_split, (p.K >> 6) - r.kb0);
  return r;
}

// tmW: weight map (128-row boxes); tmX: activation map with 128-row boxes; tmO: fp32 output
// map (128-column x 64-row boxes).  Launched as clusters of 2 CTAs; cluster i walks pair
// tiles i, i + clusters, ...
__global__ void __launch_bounds__(192, 1)
    k_gemm_tc2(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
               const __grid_constant__ CUtensorMap tmO, GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *epi = reinterpret_cast<float *>(smem + STAGES * STAGE);  // [2][64][128]
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE + 2 * EPI);
  uint64_t *peer_full = full + STAGES;  // CTA 0: CTA 1's copies of the stage have landed
  uint64_t *empty = peer_full + STAGES;
  uint64_t *acc_full = empty + STAGES;  // [2]
  uint64_t *acc_empty = acc_full + 2;   // [2], CTA 0: both CTAs' epilogues have drained it
  uint64_t *drain = acc_empty + 2;      // CTA 0: every MMA of this CTA pair has completed
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the pair protocol needs both CTAs: a launch without the cluster shape does nothing
  if (cluster_ctas() != 2) {
    if (threadIdx.x == 0) set_error(p.ctl, DEVERR_BOUNDS, 120);
    return;
  }
  const uint32_t rank = cta_rank();
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  const int ntiles = p.m_tiles * (p.n_tiles >> 1) * p.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&peer_full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc2(tmem_slot, TMEM_COLS);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers are initialised before anything targets them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      uint32_t it = 0;
      bool ok = true;
      for (int t = cid; t < ntiles && ok; t += ncl) {
        const Tile2 ti = tile2_at(p, t);
        for (int i = 0; i < ti.nkb; ++i, ++it) {
          const int s = it % STAGES;
          if (it >= (uint32_t)STAGES && !wait_c(&empty[s], ((it / STAGES) & 1) ^ 1, p.ctl, 121)) {
            ok = false;
            break;
          }
          uint8_t *st = smem + s * STAGE;
          mbar_arrive_expect_tx(&full[s], STAGE);
          tma_load_2d(st, &tmW, &full[s], (ti.kb0 + i) * 64, p.w_row0 + ti.n0 + 128 * (int)rank, pol_w);
          tma_load_2d(st + A_BYTES, &tmX, &full[s], (ti.kb0 + i) * 64, ti.m0 + 128 * (int)rank, pol_x);
        }
      }
      // every copy issued into this CTA must land before it may exit
      const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
      for (uint32_t j = first; j < it; ++j) wait_c(&full[j % STAGES], (j / STAGES) & 1, p.ctl, 122, 200000000ull);
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 1) {
      // relay: a stage of this CTA is complete -> tell the MMA issuer in CTA 0
      uint32_t it = 0;
      bool ok = true;
      for (int t = cid; t < ntiles && ok; t += ncl) {
        const Tile2 ti = tile2_at(p, t);
        for (int i = 0; i < ti.nkb; ++i, ++it) {
          const int s = it % STAGES;
          if (!wait_c(&full[s], (it / STAGES) & 1, p.ctl, 123)) {
            ok = false;
            break;
          }
          remote_arrive(cluster_addr(&peer_full[s], 0));
        }
      }
    } else if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(256, 256);
      uint32_t it = 0;
      int local = 0;
      bool ok = true;
      for (int t = cid; t < ntiles && ok; t += ncl, ++local) {
        const Tile2 ti = tile2_at(p, t);
        const int b = local & 1;
        // both epilogues must have drained this accumulator (used two tiles ago)
        if (local >= 2 && !wait_c(&acc_empty[b], ((local >> 1) & 1) ^ 1, p.ctl, 124)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * 256);
        for (int i = 0; i < ti.nkb; ++i, ++it) {
          const int s = it % STAGES;
          if (!wait_c(&full[s], (it / STAGES) & 1, p.ctl, 125) ||
              !wait_c(&peer_full[s], (it / STAGES) & 1, p.ctl, 126)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(smem + s * STAGE);
          const uint32_t bx = a + A_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma2_bf16(d, sdesc_k128(a + 32 * k), sdesc_k128(bx + 32 * k), idesc, (i > 0 || k > 0) ? 1u : 0u);
          commit2(cluster_addr(&empty[s], 0));
          commit2(cluster_addr(&empty[s], 1));
        }
        if (ok) {
          commit2(cluster_addr(&acc_full[b], 0));
          commit2(cluster_addr(&acc_full[b], 1));
        }
      }
      // no MMA of the pair may still be running when either CTA leaves
      commit2(cluster_addr(drain, 0));
      wait_c(drain, 0, p.ctl, 127, 200000000ull);
    }
  } else {
    // epilogue: warp (2..5) & 3 selects the TMEM lane quadrant (weight rows) it may access
    const int q = warp & 3;
    const int nl = q * 32 + lane;
    const bool leader = warp == 2 && lane == 0;
    const uint32_t empty0 = leader ? cluster_addr(&acc_empty[0], 0) : 0u;
    const uint32_t empty1 = leader ? cluster_addr(&acc_empty[1], 0) : 0u;
    int local = 0;
    uint32_t nbox = 0;
    for (int t = cid; t < ntiles; t += ncl, ++local) {
      const Tile2 ti = tile2_at(p, t);
      const int b = local & 1;
      if (!wait_c(&acc_full[b], (local >> 1) & 1, p.ctl, 128)) break;
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(b * 256) + ((uint32_t)(q * 32) << 16);
      const int row0 = ti.n0 + 128 * (int)rank;  // this CTA's first output feature
      const float sc = p.col_scale ? p.col_scale[row0 + nl] : 1.0f;
      for (int c0 = 0; c0 < 256 && ti.m0 + c0 < p.M; c0 += 64, ++nbox) {
        float *box = epi + (nbox & 1) * (64 * 128);
        if (leader && nbox >= 2) bulk_wait_read<1>();  // the copy that last read this box is done
        asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll 1
        for (int c = c0; c < c0 + 64; c += 32) {
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
        fence_proxy_async_shared();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (leader) {
          if (p.atomic)
            tma_reduce_add_2d(&tmO, box, row0, ti.m0 + c0);
          else
            tma_store_2d(&tmO, box, row0, ti.m0 + c0);
          bulk_commit();
        }
      }
      // this CTA's half of the accumulator has been read: tell the MMA issuer in CTA 0
      tc_fence_before();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (leader) remote_arrive(b ? empty1 : empty0);
    }
    if (leader) bulk_wait0();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the other may still reach its shared memory or TMEM
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc2(tmem, TMEM_COLS);
  }
}

}  // namespace g2

namespace {
int g_pair_clusters = 0;  // 2-CTA clusters that fit at once (0: the pair kernel is not used)
}

cudaError_t gemm2_init_attributes(int sm_count) {
  cudaError_t e = cudaFuncSetAttribute(g2::k_gemm_tc2, cudaFuncAttributeMaxDynamicSharedMemorySize, g2::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)(sm_count & ~1));
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = g2::SMEM;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, (void *)g2::k_gemm_tc2, &cfg) != cudaSuccess) {
    cudaGetLastError();
    clusters = 0;
  }
  g_pair_clusters = clusters < sm_count / 2 ? clusters : sm_count / 2;
  // opt-in: measured on B200 the pair form runs at about half the rate of the one-SM form
  // (a stage's copies complete ~3.5 us after issue and a remote arrive takes ~0.8 us to be
  // seen, so the 5-stage ring delivers one K block per ~1 us against ~0.65 us per K block in
  // the one-SM form), so the one-SM form is the default
  const char *env = std::getenv("RTVLA_PAIR_GEMM");
  if (env == nullptr || env[0] != '1') g_pair_clusters = 0;
  return cudaSuccess;
}

int gemm2_clusters() { return g_pair_clusters; }

cudaError_t gemm2_launch(const CUtensorMap &tmW, const CUtensorMap &tmX128, const CUtensorMap &tmO,
                         const GemmParams &p, cudaStream_t st) {
  const int tiles = p.m_tiles * (p.n_tiles >> 1) * p.splits;
  const int clusters = tiles < g_pair_clusters ? tiles : g_pair_clusters;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)(2 * clusters));
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = g2::SMEM;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, g2::k_gemm_tc2, tmW, tmX128, tmO, p);
}

}  // namespace rtvla
