// Multi-query attention over [valid prefix keys ; suffix keys] on the 5th-generation tensor
// cores (Realtime-VLA tech blog, kernel list "softmax_kernel_prefix_suffix": the prefix KV
// cache joined with the decoder's own K/V, the valid prefix length read at run time).
//
// One CTA = one sample, 16 queries x all 8 query heads = 128 MMA rows (row = head * 16 +
// query; the heads share the one KV head), one split of the key chunks.  Keys come in chunks
// of 64: the prefix chunks cover [0, Lv_b), the suffix chunks [0, n_suf); keys past a
// chunk's valid count are zero-filled and masked, so padded cache slots are never read.
//   S = Q K^T     tcgen05.mma M = 128, N = 64 keys, K = 256 (16 MMAs), into one of two TMEM
//                 buffers of 64 columns
//   softmax       one thread per row reads its S row from TMEM; online max with lazy
//                 rescaling: O (TMEM) is rescaled only when a row's max grows by more than
//                 2^8, otherwise P = 2^(s - m) uses the older max (P <= 2^8)
//   O += P V      tcgen05.mma M = 128, N = 256 (head dim), K = 64 keys, P from shared memory
//                 (K-major), V in its row-major [key][dim] layout as an MN-major operand
// Warps 0-3: softmax and output (warp w reads TMEM lanes 32w..32w+31); warps 4-7: loaders
// (16-byte cp.async copies into the 128-byte-swizzled operand layout, then a proxy fence;
// warps 4-5 stage K, 6-7 V); warp 8: TMEM owner, lane 0 issues the MMAs.  Splits are merged
// by k_attn_combine.  Every wait is bounded (DevCtl::timeout_ns).
#include "common.cuh"
#include "kernels.h"

namespace rtvla {
namespace atc {

constexpr int HD = 256, NH = 8, QB = 16, KC = 64;
constexpr int ROWS = NH * QB;               // 128 MMA rows
constexpr int Q_BYTES = 4 * ROWS * 128;     // 4 column blocks of [128 rows][64 bf16]
constexpr int KV_BYTES = 4 * KC * 128;      // 4 column blocks of [64 keys][64 bf16]
constexpr int P_BYTES = ROWS * 128;         // [128 rows][64 keys] bf16
constexpr int THREADS = 288;
constexpr int NBAR = 17;
constexpr int SMEM = Q_BYTES + 4 * KV_BYTES + 2 * P_BYTES + 1024 + NBAR * 8 + 16;
static_assert(SMEM <= 232448, "shared memory per CTA");
constexpr float RESCALE_LOG2 = 8.f;
constexpr uint32_t TMEM_COLS = 512;         // S buffers at columns 0 and 64, O at 128..383

// 16-byte chunk c (0..7) of row r in a [rows][128 B] tile with 128-byte swizzle
__device__ __forceinline__ uint32_t swz(uint32_t base, int r, int c) {
  return base + (uint32_t)(r * 128) + ((uint32_t)((c ^ (r & 7)) << 4));
}
// 16-byte global -> shared copy; src_bytes = 0 fills the 16 bytes with zeros
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void st_shared16(uint32_t addr, const uint4 &v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
// Shared-memory descriptor of an MN-major operand written with 128-byte swizzle: rows of
// 128 bytes along K (8-row groups 1024 bytes apart), blocks of 64 elements along MN `lbo`
// bytes apart.
__device__ __forceinline__ uint64_t sdesc_mn128(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// 32 lanes x 32 consecutive f32 columns from registers (thread i of the warp -> lane base + i)
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// The keys of chunk c of sample b: a source row pointer base and the number of valid keys.
struct Chunk {
  const bf16 *k, *v;  // key 0 of the chunk (rows of 256 bf16)
  int nvalid;
};
__device__ __forceinline__ Chunk chunk_at(const AttnParams &p, const bf16 *kpre, const bf16 *vpre, int lv, int npc,
                                          int b, int c) {
  Chunk ch;
  if (c < npc) {
    ch.k = kpre + (size_t)c * KC * HD;
    ch.v = vpre + (size_t)c * KC * HD;
    ch.nvalid = min(KC, lv - c * KC);
  } else {
    const int c2 = c - npc;
    const size_t off = ((size_t)b * p.n_suf + (size_t)c2 * KC) * HD;
    ch.k = p.ksuf + off;
    ch.v = p.vsuf + off;
    ch.nvalid = min(KC, p.n_suf - c2 * KC);
  }
  return ch;
}

__global__ void __launch_bounds__(THREADS, 1) k_attn_tc(AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t qs = smem_u32(smem);
  const uint32_t ks0 = qs + Q_BYTES, vs0 = qs + Q_BYTES + 2 * KV_BYTES, ps0 = qs + Q_BYTES + 4 * KV_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Q_BYTES + 4 * KV_BYTES + 2 * P_BYTES);
  uint64_t *q_full = bars;          // loaders -> MMA: Q staged
  uint64_t *k_full = bars + 1;      // [2] K loaders -> MMA: a chunk's K staged
  uint64_t *k_empty = bars + 3;     // [2] MMA -> K loaders: the chunk's S MMAs are done
  uint64_t *v_full = bars + 5;      // [2] V loaders -> MMA: a chunk's V staged
  uint64_t *v_empty = bars + 7;     // [2] MMA -> V loaders: the chunk's PV MMAs are done
  uint64_t *s_full = bars + 9;      // [2] MMA -> softmax: S in TMEM
  uint64_t *s_empty = bars + 11;    // [2] softmax -> MMA: S read
  uint64_t *p_full = bars + 13;     // [2] softmax -> MMA: P written (and O rescaled)
  uint64_t *p_empty = bars + 15;    // [2] MMA -> softmax: PV done (P buffer free, O current)
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(p_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, qb = blockIdx.y, b = blockIdx.z;
  const CallArgs *ca = p.ca;
  const int B = ca->batch, cap = ca->cap;
  int lv = ca->valid_len[b];
  if (lv < 0 || lv > cap) {
    if (threadIdx.x == 0 && split == 0 && qb == 0) set_error(p.ctl, DEVERR_BOUNDS, 211);
    lv = lv < 0 ? 0 : cap;
  }
  const size_t lay = (size_t)p.layer * B * cap * HD + (size_t)b * cap * HD;
  const bf16 *kpre = ca->kv_k + lay;
  const bf16 *vpre = ca->kv_v + lay;
  const int npc = (lv + KC - 1) / KC, nsc = (p.n_suf + KC - 1) / KC;
  const int cps = p.keys_per_split / KC;
  const int c_begin = split * cps;
  const int c_end = min(npc + nsc, c_begin + cps);
  const int nch = c_end > c_begin ? c_end - c_begin : 0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 64);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 64);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&p_empty[i], 1);
    }
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------------ loaders
    // 16-byte cp.async copies straight into the swizzled operand layout (zero-filled where a
    // key or query does not exist); each thread waits for its own copies, fences them to the
    // async proxy and arrives.  Warps 4-5 stage K, warps 6-7 stage V, each on its own pair of
    // buffers: K of chunk i + 2 is requested once S of chunk i is done, V once its PV is.
    const int lt = threadIdx.x - 128;
    // Q: 128 rows x 32 chunks of 16 bytes; rows of queries past nq are zero
#pragma unroll 4
    for (int i = 0; i < 32; ++i) {
      const int idx = lt + 128 * i;
      const int r = idx >> 5, cc = idx & 31;
      const int q = qb * QB + (r & 15);
      const bool ok = q < p.nq;
      const bf16 *src = p.q + (size_t)(b * p.nq + (ok ? q : 0)) * p.q_ld + (r >> 4) * HD + cc * 8;
      cp_async16(swz(qs + (cc >> 3) * (ROWS * 128), r, cc & 7), src, ok ? 16u : 0u);
    }
    cp_async_commit();
    cp_async_wait_all();
    fence_proxy_async_shared();
    mbar_arrive(q_full);
    const bool is_k = warp < 6;
    const int gt = lt & 63;  // thread within the K or the V group
    uint64_t *full = is_k ? k_full : v_full;
    uint64_t *empty = is_k ? k_empty : v_empty;
#pragma unroll 1
    for (int i = 0; i < nch; ++i) {
      const int bb = i & 1;
      if (i >= 2 && !mbar_wait(&empty[bb], ((i >> 1) & 1) ^ 1, p.ctl, 212)) break;
      const Chunk ch = chunk_at(p, kpre, vpre, lv, npc, b, c_begin + i);
      const uint32_t dst = (is_k ? ks0 : vs0) + bb * KV_BYTES;
      const bf16 *src = is_k ? ch.k : ch.v;
#pragma unroll 8
      for (int m = 0; m < 32; ++m) {
        const int idx = gt + 64 * m;
        const int j = idx >> 5, cc = idx & 31;
        const bool ok = j < ch.nvalid;
        cp_async16(swz(dst + (cc >> 3) * (KC * 128), j, cc & 7), src + (size_t)(ok ? j : 0) * HD + cc * 8,
                   ok ? 16u : 0u);
      }
      cp_async_commit();
      cp_async_wait_all();
      fence_proxy_async_shared();
      mbar_arrive(&full[bb]);
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && nch > 0) {
      constexpr uint32_t idesc_s = idesc_bf16(ROWS, KC);
      constexpr uint32_t idesc_pv = idesc_bf16(ROWS, HD) | (1u << 16);  // B (V) MN-major
      bool ok = mbar_wait(q_full, 0, p.ctl, 213);
      auto issue_s = [&](int i) -> bool {
        const int bb = i & 1;
        if (!mbar_wait(&k_full[bb], (i >> 1) & 1, p.ctl, 214)) return false;
        if (i >= 2 && !mbar_wait(&s_empty[bb], ((i >> 1) & 1) ^ 1, p.ctl, 215)) return false;
        tc_fence_after();
        const uint32_t kb0 = ks0 + bb * KV_BYTES;
#pragma unroll
        for (int kb = 0; kb < 4; ++kb)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tmem + (uint32_t)(bb * KC), sdesc_k128(qs + kb * (ROWS * 128) + 32 * k),
                      sdesc_k128(kb0 + kb * (KC * 128) + 32 * k), idesc_s, (kb | k) ? 1u : 0u);
        umma_commit(&s_full[bb]);
        umma_commit(&k_empty[bb]);
        return true;
      };
      if (ok) ok = issue_s(0);
#pragma unroll 1
      for (int i = 0; i < nch && ok; ++i) {
        if (i + 1 < nch && !issue_s(i + 1)) break;
        const int bb = i & 1;
        if (!mbar_wait(&p_full[bb], (i >> 1) & 1, p.ctl, 216) || !mbar_wait(&v_full[bb], (i >> 1) & 1, p.ctl, 221))
          break;
        tc_fence_after();
        const uint32_t pa = ps0 + bb * P_BYTES, va = vs0 + bb * KV_BYTES;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tmem + 2 * KC, sdesc_k128(pa + 32 * k), sdesc_mn128(va + k * 16 * 128, KC * 128), idesc_pv,
                    (i > 0 || k > 0) ? 1u : 0u);
        umma_commit(&p_empty[bb]);
        umma_commit(&v_empty[bb]);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax and output
    const int r = warp * 32 + lane;  // MMA row = TMEM lane
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
#pragma unroll 1
    for (int i = 0; i < nch && ok; ++i) {
      const int bb = i & 1;
      const Chunk ch = chunk_at(p, kpre, vpre, lv, npc, b, c_begin + i);
      if (!mbar_wait(&s_full[bb], (i >> 1) & 1, p.ctl, 217)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[64];
      {
        float lo[32], hi[32];
        tmem_ld32(trow + (uint32_t)(bb * KC), lo);
        tmem_ld32(trow + (uint32_t)(bb * KC + 32), hi);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          s[j] = j < ch.nvalid ? lo[j] * p.scale_log2 : -INFINITY;
          s[32 + j] = 32 + j < ch.nvalid ? hi[j] * p.scale_log2 : -INFINITY;
        }
      }
      tc_fence_before();
      mbar_arrive(&s_empty[bb]);
      float cm = -INFINITY;
#pragma unroll
      for (int j = 0; j < 64; ++j) cm = fmaxf(cm, s[j]);
      // every chunk has at least one valid key, so cm is finite
      const bool resc = m != -INFINITY && cm > m + RESCALE_LOG2;
      if (__any_sync(0xffffffffu, resc)) {
        // O holds the sum up to chunk i - 1: wait for that PV, rescale the rows whose max grew
        if (!mbar_wait(&p_empty[(i - 1) & 1], ((i - 1) >> 1) & 1, p.ctl, 218)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float alpha = resc ? exp2f(m - cm) : 1.f;
#pragma unroll 1
        for (int q = 0; q < 8; ++q) {
          float o[32];
          tmem_ld32(trow + (uint32_t)(2 * KC + 32 * q), o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(trow + (uint32_t)(2 * KC + 32 * q), o);
        }
        tc_fence_before();
        l *= alpha;
      }
      if (m == -INFINITY || resc) m = cm;
      // the P buffer was last read by the PV of chunk i - 2
      if (i >= 2 && !mbar_wait(&p_empty[bb], ((i >> 1) & 1) ^ 1, p.ctl, 219)) {
        ok = false;
        break;
      }
      const uint32_t prow = ps0 + bb * P_BYTES;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        float e[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          e[u] = exp2f(s[c8 * 8 + u] - m);  // masked keys: 2^-inf = 0
          l += e[u];
        }
        uint4 v;
        v.x = pack_bf16(e[0], e[1]);
        v.y = pack_bf16(e[2], e[3]);
        v.z = pack_bf16(e[4], e[5]);
        v.w = pack_bf16(e[6], e[7]);
        st_shared16(swz(prow, r, c8), v);
      }
      fence_proxy_async_shared();
      mbar_arrive(&p_full[bb]);
    }
    // ---- output: this row's 256 values of O
    const int h = r >> 4, q = qb * QB + (r & 15);
    const bool have = ok && nch > 0 &&
                      mbar_wait(&p_empty[(nch - 1) & 1], ((nch - 1) >> 1) & 1, p.ctl, 220);
    if (have) tc_fence_after();
    const bool single = p.n_splits == 1;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const size_t base = ((size_t)b * p.n_splits + split) * p.nq;
#pragma unroll 1
    for (int cb = 0; cb < 8; ++cb) {
      float o[32];
      if (have) {
        tmem_ld32(trow + (uint32_t)(2 * KC + 32 * cb), o);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0.f;
      }
      if (q < p.nq) {
        if (single) {
          bf16 *dst = p.out + (size_t)(b * p.nq + q) * (NH * HD) + h * HD + cb * 32;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 v;
            v.x = pack_bf16(o[8 * u] * inv, o[8 * u + 1] * inv);
            v.y = pack_bf16(o[8 * u + 2] * inv, o[8 * u + 3] * inv);
            v.z = pack_bf16(o[8 * u + 4] * inv, o[8 * u + 5] * inv);
            v.w = pack_bf16(o[8 * u + 6] * inv, o[8 * u + 7] * inv);
            *reinterpret_cast<uint4 *>(dst + 8 * u) = v;
          }
        } else {
          float *dst = p.opart + ((base + q) * NH + h) * HD + cb * 32;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<float4 *>(dst + 4 * u) = make_float4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
        }
      }
    }
    if (!single && q < p.nq)
      *reinterpret_cast<float2 *>(p.mlpart + ((base + q) * NH + h) * 2) = make_float2(have ? m : -INFINITY, have ? l : 0.f);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace atc

cudaError_t attn_tc_init_attributes() {
  return cudaFuncSetAttribute(atc::k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, atc::SMEM);
}

cudaError_t attn_tc_launch(const AttnParams &p, int batch, cudaStream_t st) {
  dim3 grid(p.n_splits, (p.nq + atc::QB - 1) / atc::QB, batch);
  atc::k_attn_tc<<<grid, atc::THREADS, atc::SMEM, st>>>(p);
  return cudaGetLastError();
}

}  // namespace rtvla
