// Persistent engine: the whole 10-step denoise loop as ONE cooperative kernel (batch 1,
// chunk <= 64), one CTA per SM.
//
// The loop is weight-streaming bound (622 MB of bf16 expert weights per Euler step) and is
// a chain of dependent phases per layer.  Weights never depend on activations, so:
//   warp 0     TMA producer: walks this CTA's static list of weight tiles for every GEMM of
//              the whole loop and keeps a 5-stage shared-memory ring full, never waiting on
//              an activation; it also prefetches the next phase's table slices into L2;
//   warp 1     tcgen05 MMA issuer (accumulator in TMEM), started per 64-wide K block as soon
//              as that block of the activation operand is in shared memory;
//   warps 2..9 compute: stage activations with TMA (fp32 tiles, 128-byte swizzle, four
//              per 3-D box) and turn them into the bf16 operand (fused AdaRMS modulation / GELU(gate) * up), run
//              the epilogue (TMEM -> shared tile -> one TMA bulk reduce-add into fp32; the
//              AdaRMS gate of the residual applied on the way), and run the Q/K/V finalise,
//              attention, split merge and final / Euler phases; a grid barrier separates
//              phases.
// Activations written by one CTA and read by many are read through the TMA / bulk-copy
// engine, not per-thread loads: the bulk engine keeps far more bytes in flight per SM.
// The CUDA-graph realisation of the same loop is the layered engine (rtvla_api.cu); this file
// is the persistent-kernel alternative to the Realtime-VLA tech blog's CUDA-graph replay,
// with the launch gaps of ~1800 kernels replaced by grid barriers under which the weight
// stream continues.
#include "common.cuh"
#include "kernels.h"
#include "persistent.h"

namespace rtvla {
namespace pk {

constexpr int THREADS = 320;
constexpr int NCOMP = 256;
constexpr int RING = 5;
constexpr int WST = 128 * 128;            // one 128-row x 64-column bf16 weight tile
constexpr int NOPK = 8;                   // operand K blocks (64 tokens x 64 bf16 each, 128B swizzle)
constexpr int OPB = NOPK * 8192;
constexpr int NGRP = 2;                   // fp32 staging groups (double buffer)
constexpr int STG = 8192;                 // one staged tile: 64 rows x 32 columns, 128B swizzle
constexpr int GRPB = 4 * STG;             // a group: 4 tiles, filled by one or two 3-D TMA boxes
constexpr int TBL = 4096;                 // per-unit slice of the AdaRMS scale / GELU bias tables
constexpr int REGION = OPB + NGRP * GRPB + TBL;  // operands + staging + table | attention | epilogue tile
constexpr int LDS = 264;                  // attention shared rows (bf16), 528 bytes
constexpr int KC = 32;                    // attention keys per chunk
constexpr int ATT_BYTES = (64 + 2 * KC) * LDS * 2;
static_assert(ATT_BYTES <= REGION, "attention tiles must fit the shared region");
constexpr int NBARS = 2 * RING + NOPK + NGRP + 4;
constexpr int SMEM = RING * WST + REGION + 1024 + NBARS * 8 + 64;
constexpr int D = 1024, F = 4096, HD = 256, NH = 8, A = 32;
constexpr int MAXSPLIT = 18;

enum Kind { QKV = 0, OPJ = 1, GU = 2, DN = 3 };
// N tiles (128 output features), 64-wide K blocks, K splits per GEMM kind
__device__ __forceinline__ int n_tiles(int kind) { return kind == QKV ? 20 : (kind == GU ? 64 : 8); }
__device__ __forceinline__ int kb_total(int kind) { return kind == QKV || kind == GU ? 16 : (kind == OPJ ? 32 : 64); }
__device__ __forceinline__ int k_splits(int kind) { return kind == QKV ? 7 : (kind == GU ? 2 : 18); }
__device__ __forceinline__ int units(int kind) { return n_tiles(kind) * k_splits(kind); }
__device__ __forceinline__ int rows_per_layer(int kind) { return kind == QKV ? 2560 : (kind == GU ? 8192 : 1024); }
__device__ __forceinline__ int rotation(int gp, int ncta) { return (gp * 37) % ncta; }
__device__ __forceinline__ int first_unit(int gp, int c, int ncta) {
  return (c - rotation(gp, ncta) + ncta) % ncta;
}
__device__ __forceinline__ void unit_kb(int kind, int u, int &nt, int &kb0, int &kb1) {
  const int T = n_tiles(kind), S = k_splits(kind), K = kb_total(kind);
  nt = u % T;
  const int s = u / T;
  kb0 = s * K / S;
  kb1 = (s + 1) * K / S;
}

__device__ __forceinline__ void named_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ unsigned ld_relaxed(const unsigned *p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int aborted(DevCtl *ctl) { return *reinterpret_cast<volatile int *>(&ctl->err); }

// mbarrier wait that also gives up as soon as any CTA has recorded an error.  Drains (copies
// or MMAs that must land before the CTA exits) ignore the abort flag and wait at least 200 ms
// whatever the configured limit.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, DevCtl *ctl, int where,
                                         bool stop_on_abort = true) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  uint64_t lim = ctl->timeout_ns;
  if (!stop_on_abort && lim < 200000000ull) lim = 200000000ull;
#pragma unroll 1
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(a, parity)) return true;
    if ((i & 255) == 0) {
      if (stop_on_abort && aborted(ctl)) return false;
      if (globaltimer() - t0 > lim) {
        set_error(ctl, DEVERR_TIMEOUT, where);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void stamp(const PersistParams &p, unsigned epoch, int slot) {
  if (p.stamps != nullptr && (int)epoch < p.max_phases)
    p.stamps[((size_t)blockIdx.x * p.max_phases + epoch) * 8 + slot] = globaltimer();
}

// Grid barrier among the compute warps of all CTAs.  Arrivals are spread over NBC monotone
// counters (CTA c adds to counter c % NBC, 128 bytes apart) so that they do not queue on one
// address; a CTA passes when every counter has reached its share of the epoch.  The counters
// are zeroed by the per-call argument copy.  Thread 0 first waits for this CTA's bulk
// reductions, so everything the CTA wrote in the phase is visible (to the generic and the
// async proxy) once the barrier opens.
constexpr int NBC = 2;  // measured on B200: 2 beat 8 by ~0.06 ms per call (and 1, 4 by less)
// relaxed polls of all counters in flight together; the caller's fence gives acquire order
__device__ __forceinline__ bool bar_passed(const unsigned *bar, unsigned epoch, int ncta) {
  unsigned v[NBC];
#pragma unroll
  for (int i = 0; i < NBC; ++i) v[i] = ld_relaxed(bar + 32 * i);
  bool ok = true;
#pragma unroll
  for (int i = 0; i < NBC; ++i) ok &= v[i] >= epoch * (unsigned)((ncta - i + NBC - 1) / NBC);
  return ok;
}
__device__ __forceinline__ void grid_sync(const PersistParams &p, unsigned *bar, DevCtl *ctl, unsigned &epoch,
                                          int ncta, int tid) {
  named_sync();
  if (tid == 0) {
    bulk_wait0();
    fence_proxy_async_global();
    stamp(p, epoch, 7);
    ++epoch;
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(bar + 32 * (blockIdx.x % NBC)) : "memory");
    if (!bar_passed(bar, epoch, ncta)) {
      const uint64_t t0 = globaltimer();
      const uint64_t lim = ctl->timeout_ns;
#pragma unroll 1
      for (uint32_t i = 1;; ++i) {
        if (bar_passed(bar, epoch, ncta)) break;
        if ((i & 63) == 0) {
          if (aborted(ctl)) break;
          if (globaltimer() - t0 > lim) {
            set_error(ctl, DEVERR_TIMEOUT, 601);
            break;
          }
        }
      }
    }
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    fence_proxy_async_global();
    stamp(p, epoch, 0);
  }
  named_sync();
}

__device__ __forceinline__ void zero_slice(float *buf, size_t n, int c, int ncta, int tid) {
  const size_t per = ((n + (size_t)ncta - 1) / ncta + 3) & ~size_t(3);
  const size_t b = (size_t)c * per, e = b + per < n ? b + per : n;
  for (size_t i = b + (size_t)tid * 4; i < e; i += NCOMP * 4) {
    if (i + 4 <= e)
      *reinterpret_cast<float4 *>(buf + i) = make_float4(0, 0, 0, 0);
    else
      for (size_t j = i; j < e; ++j) buf[j] = 0.f;
  }
}

// ---------------------------------------------------------------------------------------
// shared-memory state

struct Smem {
  uint8_t *ring, *op, *stg;
  float *tbl;
  uint64_t *full, *empty, *opf, *stgb, *acc_ready, *drain, *att, *tblb;
  uint32_t *tmem_slot;
};

// 8 consecutive fp32 of row r (logical 16-byte chunks c, c+1) of a 64 x 32 staging tile
// written by TMA with 128-byte swizzle (16-byte chunk c of row r sits at c ^ (r & 7))
__device__ __forceinline__ void stg_read8(const uint8_t *t, int r, int c, float *v) {
  const float4 a = *reinterpret_cast<const float4 *>(t + r * 128 + ((c ^ (r & 7)) << 4));
  const float4 b = *reinterpret_cast<const float4 *>(t + r * 128 + (((c + 1) ^ (r & 7)) << 4));
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
// the 16-byte chunk cc (0..7) of operand row r in K block j (128-byte swizzle)
__device__ __forceinline__ uint4 *op_chunk(uint8_t *op, int j, int r, int cc) {
  return reinterpret_cast<uint4 *>(op + j * 8192 + r * 128 + ((cc ^ (r & 7)) << 4));
}

// Builds the bf16 operand of one GEMM unit from fp32 tiles staged by TMA and releases each
// 64-wide K block to the MMA as soon as it is complete.  Staging runs in groups of four
// 64-row x 32-column tiles, double-buffered: QKV / GU fetch a group as one 3-D box of four
// consecutive column tiles of h; DN as two boxes (two gate tiles, the two matching up tiles).
// One wait, one proxy fence and one barrier per group; the group after next is issued as soon
// as a buffer is consumed.
//   QKV / GU:  bf16(h * (1 + scale)); designated units add the slice's sum of squares of h
//   DN:        bf16(GELU_tanh(r*g + bg) * (r*u + bu)) from the gate/up accumulator
__device__ void build_operand(const PersistParams &p, const Smem &sm, const CUtensorMap *tm_lh,
                              const CUtensorMap *tm_lg, int kind, int kb0, int nkb, const float *s1p,
                              const float *bias, float *ss, bool stats, int M, uint32_t &g, uint32_t &ntbl,
                              int tid) {
  const bool dn = kind == DN;
  const int npieces = 2 * nkb;          // 32-column pieces of the unit's K slice
  const int ppg = dn ? 2 : 4;           // pieces per group
  const int ngroups = (npieces + ppg - 1) / ppg;
  const uint32_t g0 = g;
  const int ncol = nkb * 64;            // table slice: scale (QKV, GU) or gate | up bias (DN)
  uint64_t pol = 0;
  // group q covers pieces [q * ppg, q * ppg + ppg) (a short last group reads its box's spare
  // tiles from the neighbouring columns, or zero fill past the end; they are never used)
  auto issue = [&](int q) {
    const int buf = (g0 + q) % NGRP;
    uint8_t *dst = sm.stg + buf * GRPB;
    const int z = (kb0 * 64) / 32 + q * ppg;
    mbar_arrive_expect_tx(&sm.stgb[buf], GRPB);
    if (dn) {
      tma_load_3d(dst, tm_lg, &sm.stgb[buf], 0, 0, z, pol);
      tma_load_3d(dst + 2 * STG, tm_lg, &sm.stgb[buf], 0, 0, z + F / 32, pol);
    } else {
      tma_load_3d(dst, tm_lh, &sm.stgb[buf], 0, 0, z, pol);
    }
  };
  if (tid == 0) {
    pol = policy_evict_last();
    for (int q = 0; q < ngroups && q < NGRP; ++q) issue(q);
    if (dn) {
      mbar_arrive_expect_tx(sm.tblb, 2 * ncol * 4);
      bulk_load(sm.tbl, bias + kb0 * 64, ncol * 4, sm.tblb);
      bulk_load(sm.tbl + ncol, bias + F + kb0 * 64, ncol * 4, sm.tblb);
    } else {
      mbar_arrive_expect_tx(sm.tblb, ncol * 4);
      bulk_load(sm.tbl, s1p + kb0 * 64, ncol * 4, sm.tblb);
    }
  }
  const int r = tid >> 2, sub = tid & 3;
  float acc = 0.f;
  float rr = 0.f;
  if (dn && r < M) rr = rsqrtf(__ldcg(ss + r) * (1.0f / D) + p.eps);
  wait_bar(sm.tblb, ntbl & 1, p.ctl, 642);
  ++ntbl;
  for (int q = 0; q < ngroups; ++q) {
    const uint32_t gq = g0 + q;
    const uint8_t *grp = sm.stg + (gq % NGRP) * GRPB;
    wait_bar(&sm.stgb[gq % NGRP], (gq / NGRP) & 1, p.ctl, 641);
    const int p0 = q * ppg, pe = p0 + ppg < npieces ? p0 + ppg : npieces;
    for (int pc = p0; pc < pe; ++pc) {
      const int col = pc * 32 + sub * 8;  // column within the unit's K slice
      const int j = pc >> 1, cc = (pc & 1) * 4 + sub;
      uint4 out = make_uint4(0, 0, 0, 0);
      if (r < M) {
        float v[8];
        if (dn) {
          float u[8];
          stg_read8(grp + (pc - p0) * STG, r, 2 * sub, v);
          stg_read8(grp + (2 + pc - p0) * STG, r, 2 * sub, u);
          const float4 bg0 = *reinterpret_cast<const float4 *>(sm.tbl + col);
          const float4 bg1 = *reinterpret_cast<const float4 *>(sm.tbl + col + 4);
          const float4 bu0 = *reinterpret_cast<const float4 *>(sm.tbl + ncol + col);
          const float4 bu1 = *reinterpret_cast<const float4 *>(sm.tbl + ncol + col + 4);
          const float bgv[8] = {bg0.x, bg0.y, bg0.z, bg0.w, bg1.x, bg1.y, bg1.z, bg1.w};
          const float buv[8] = {bu0.x, bu0.y, bu0.z, bu0.w, bu1.x, bu1.y, bu1.z, bu1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = gelu_tanh_fast(rr * v[e] + bgv[e]) * (rr * u[e] + buv[e]);
        } else {
          stg_read8(grp + (pc - p0) * STG, r, 2 * sub, v);
          const float4 s0 = *reinterpret_cast<const float4 *>(sm.tbl + col);
          const float4 s1 = *reinterpret_cast<const float4 *>(sm.tbl + col + 4);
          const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            acc += v[e] * v[e];
            v[e] *= sv[e];
          }
        }
        out.x = pack_bf16(v[0], v[1]);
        out.y = pack_bf16(v[2], v[3]);
        out.z = pack_bf16(v[4], v[5]);
        out.w = pack_bf16(v[6], v[7]);
      }
      *op_chunk(sm.op, j, r, cc) = out;
    }
    fence_proxy_async_shared();  // the group's K blocks are complete: visible to the MMA
    named_sync();
    if (tid == 0) {
      for (int j = p0 >> 1; j < (pe >> 1); ++j) mbar_arrive(&sm.opf[j]);
      if (q + NGRP < ngroups) issue(q + NGRP);  // refill the buffer just consumed
    }
  }
  g = g0 + ngroups;
  if (stats) {
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (sub == 0 && r < M) atomicAdd(ss + r, acc);
  }
}

// ---------------------------------------------------------------------------------------
// Q/K/V finalise: y = r * acc + bias, RoPE at position lv + q on the 8 query heads and the
// key; bf16 Q [64][2048], K_s / V_s [64][256].  Four (row, head) tasks per pass, 64 threads
// each, every load of a pass in flight at once.

__device__ void qkv_finalise(const PersistParams &p, int lv, size_t kl, int c, int ncta, int C, int tid) {
  const float *bias = p.bias_qkv + kl * 2560;
  const int lt = tid & 31;
  for (int base = c * 8; base < C * 10; base += ncta * 8) {
    const int task = base + (tid >> 5);
    if (task >= C * 10) continue;
    const int q = task / 10, blk = task % 10;
    const float *a = p.acc_qkv + (size_t)q * 2560;
    const float rr = rsqrtf(__ldcg(p.ss_attn + q) * (1.0f / D) + p.eps);
    if (blk < 9) {
      const int col0 = blk * HD, d = lt * 4;
      const int pos = lv + q;
      const float4 x1 = __ldcg(reinterpret_cast<const float4 *>(a + col0 + d));
      const float4 x2 = __ldcg(reinterpret_cast<const float4 *>(a + col0 + 128 + d));
      const float4 co = __ldg(reinterpret_cast<const float4 *>(p.rope_cos + (size_t)pos * 128 + d));
      const float4 si = __ldg(reinterpret_cast<const float4 *>(p.rope_sin + (size_t)pos * 128 + d));
      const float4 b1 = __ldg(reinterpret_cast<const float4 *>(bias + col0 + d));
      const float4 b2 = __ldg(reinterpret_cast<const float4 *>(bias + col0 + 128 + d));
      const float u[4] = {rr * x1.x + b1.x, rr * x1.y + b1.y, rr * x1.z + b1.z, rr * x1.w + b1.w};
      const float w[4] = {rr * x2.x + b2.x, rr * x2.y + b2.y, rr * x2.z + b2.z, rr * x2.w + b2.w};
      const float cv[4] = {co.x, co.y, co.z, co.w}, sv[4] = {si.x, si.y, si.z, si.w};
      float lo[4], hi[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        lo[e] = u[e] * cv[e] - w[e] * sv[e];
        hi[e] = w[e] * cv[e] + u[e] * sv[e];
      }
      bf16 *dst = blk < 8 ? p.qb + (size_t)q * 2048 + col0 : p.ks + (size_t)q * HD;
      *reinterpret_cast<uint2 *>(dst + d) = make_uint2(pack_bf16(lo[0], lo[1]), pack_bf16(lo[2], lo[3]));
      *reinterpret_cast<uint2 *>(dst + 128 + d) = make_uint2(pack_bf16(hi[0], hi[1]), pack_bf16(hi[2], hi[3]));
    } else {
      const int d = lt * 8;
      const float4 x0 = __ldcg(reinterpret_cast<const float4 *>(a + 2304 + d));
      const float4 x1 = __ldcg(reinterpret_cast<const float4 *>(a + 2304 + d + 4));
      const float4 b0 = __ldg(reinterpret_cast<const float4 *>(bias + 2304 + d));
      const float4 b1 = __ldg(reinterpret_cast<const float4 *>(bias + 2304 + d + 4));
      uint4 v;
      v.x = pack_bf16(rr * x0.x + b0.x, rr * x0.y + b0.y);
      v.y = pack_bf16(rr * x0.z + b0.z, rr * x0.w + b0.w);
      v.z = pack_bf16(rr * x1.x + b1.x, rr * x1.y + b1.y);
      v.w = pack_bf16(rr * x1.z + b1.z, rr * x1.w + b1.w);
      *reinterpret_cast<uint4 *>(p.vs + (size_t)q * HD + d) = v;
    }
  }
}

// ---------------------------------------------------------------------------------------
// attention unit: head h, key split s; 8 warps = 4 query blocks of 16 x 2 halves of head_dim.
// Keys are taken in chunks of 32 that never mix prefix and suffix: chunks [0, npre) cover the
// valid prefix (from the cache), chunks [npre, npre + nsuf) the C suffix keys (finalised
// K_s / V_s).  Q_h and each K / V chunk arrive by TMA as four 64-column boxes with 128-byte
// swizzle (element (r, c) of a [4][R][64] tile at block c/64, row r, 16-byte chunk
// ((c%64)/8) ^ (r%8)).

struct AttnCtx {
  int lv, npre, nsuf, cps, nsplit;
};

__device__ __forceinline__ uint32_t swz_addr(uint32_t base, int rows, int r, int c) {
  return base + (c >> 6) * (rows * 128) + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1);
}

__device__ void attn_unit(const PersistParams &p, const Smem &sm, const AttnCtx &ac, int h, int s, int l,
                          const CUtensorMap *tm_q, const CUtensorMap *tm_kc, const CUtensorMap *tm_vc,
                          const CUtensorMap *tm_ks, const CUtensorMap *tm_vs, uint32_t &natt, int tid,
                          unsigned epoch) {
  uint8_t *Qs = sm.op;               // [4][64][64] bf16, swizzled
  uint8_t *Ks = sm.op + 32768;       // [4][32][64]
  uint8_t *Vs = sm.op + 49152;       // [4][32][64]
  const uint32_t qa_ = smem_u32(Qs), ka_ = smem_u32(Ks), va_ = smem_u32(Vs);
  const int warp = tid >> 5, lane = tid & 31;
  const int nch = ac.npre + ac.nsuf;
  const int ch0 = s * ac.cps, ch1 = min(nch, ch0 + ac.cps);
  const int cap = p.ca_cap;

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int g = lane >> 2, t = lane & 3;
  const int qb = warp & 3, dh = warp >> 2;

#pragma unroll 1
  for (int ch = ch0; ch < ch1; ++ch) {
    const bool pre = ch < ac.npre;
    const int nv = pre ? min(KC, ac.lv - ch * KC) : min(KC, p.C - (ch - ac.npre) * KC);
    named_sync();  // the previous chunk has been consumed
    if (tid == 0) {
      const uint64_t pol = policy_evict_last();
      const bool first = ch == ch0;
      mbar_arrive_expect_tx(sm.att, (first ? 32768u : 0u) + 32768u);
      if (first)
        for (int b = 0; b < 4; ++b) tma_load_2d(Qs + b * 8192, tm_q, sm.att, h * HD + b * 64, 0, pol);
      const CUtensorMap *mk = pre ? tm_kc : tm_ks;
      const CUtensorMap *mv = pre ? tm_vc : tm_vs;
      const int y = pre ? l * cap + ch * KC : (ch - ac.npre) * KC;
      for (int b = 0; b < 4; ++b) {
        tma_load_2d(Ks + b * 4096, mk, sm.att, b * 64, y, pol);
        tma_load_2d(Vs + b * 4096, mv, sm.att, b * 64, y, pol);
      }
    }
    wait_bar(sm.att, natt & 1, p.ctl, 651);
    ++natt;
    // rows past the chunk's valid keys may hold anything: zero them (V is multiplied by p = 0)
    for (int i = tid; i < (KC - nv) * 32; i += NCOMP) {
      const int r = nv + (i >> 5), q16 = i & 31;  // 32 x 16 bytes per row (4 blocks x 8 chunks)
      const int b = q16 >> 3, c16 = q16 & 7;
      *reinterpret_cast<uint4 *>(Ks + b * 4096 + r * 128 + (c16 << 4)) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4 *>(Vs + b * 4096 + r * 128 + (c16 << 4)) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_shared();  // these generic writes precede the next chunk's TMA writes
    named_sync();
    if (ch == ch0 && tid == 0) stamp(p, epoch, 4);

    float sc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(a0, a1, a2, a3, swz_addr(qa_, 64, qb * 16 + (lane & 15), kk * 16 + (lane >> 4) * 8));
#pragma unroll
      for (int nt = 0; nt < 4; nt += 2) {
        uint32_t b0, b1, b2, b3;
        const int r = nt * 8 + (lane & 7) + ((lane >> 4) << 3);
        const int c = kk * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4(b0, b1, b2, b3, swz_addr(ka_, 32, r, c));
        mma_16816(sc[nt], a0, a1, a2, a3, b0, b1);
        mma_16816(sc[nt + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    float cm0 = -INFINITY, cm1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = nt * 8 + 2 * t + (e & 1);
        const float v = (key < nv) ? sc[nt][e] * p.scale_log2 : -INFINITY;
        sc[nt][e] = v;
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
    for (int nt = 0; nt < 4; ++nt) {
      sc[nt][0] = exp2f(sc[nt][0] - r0);
      sc[nt][1] = exp2f(sc[nt][1] - r0);
      sc[nt][2] = exp2f(sc[nt][2] - r1);
      sc[nt][3] = exp2f(sc[nt][3] - r1);
      ps0 += sc[nt][0] + sc[nt][1];
      ps1 += sc[nt][2] + sc[nt][3];
    }
    l0 = l0 * al0 + ps0;
    l1 = l1 * al1 + ps1;
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      o[dt][0] *= al0;
      o[dt][1] *= al0;
      o[dt][2] *= al1;
      o[dt][3] *= al1;
    }
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) {
      const uint32_t a0 = pack_bf16(sc[2 * kt][0], sc[2 * kt][1]);
      const uint32_t a1 = pack_bf16(sc[2 * kt][2], sc[2 * kt][3]);
      const uint32_t a2 = pack_bf16(sc[2 * kt + 1][0], sc[2 * kt + 1][1]);
      const uint32_t a3 = pack_bf16(sc[2 * kt + 1][2], sc[2 * kt + 1][3]);
#pragma unroll
      for (int dt = 0; dt < 16; dt += 2) {
        uint32_t b0, b1, b2, b3;
        const int r = kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = dh * 128 + dt * 8 + (lane >> 4) * 8;
        ldsm_x4_t(b0, b1, b2, b3, swz_addr(va_, 32, r, c));
        mma_16816(o[dt], a0, a1, a2, a3, b0, b1);
        mma_16816(o[dt + 1], a0, a1, a2, a3, b2, b3);
      }
    }
  }
  if (tid == 0) stamp(p, epoch, 6);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const int qa = qb * 16 + g, qc = qa + 8;
  const size_t rowbase = ((size_t)s * NH + h) * 64;
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) {
    const int d = dh * 128 + dt * 8 + 2 * t;
    *reinterpret_cast<float2 *>(p.opart + (rowbase + qa) * HD + d) = make_float2(o[dt][0], o[dt][1]);
    *reinterpret_cast<float2 *>(p.opart + (rowbase + qc) * HD + d) = make_float2(o[dt][2], o[dt][3]);
  }
  if (dh == 0 && t == 0) {
    *reinterpret_cast<float2 *>(p.mlpart + (rowbase + qa) * 2) = make_float2(m0, l0);
    *reinterpret_cast<float2 *>(p.mlpart + (rowbase + qc) * 2) = make_float2(m1, l1);
  }
}

// Merges the key splits of rows (head, query) into the bf16 attention output.  Four rows at a
// time, 64 threads x 4 dims per row; the splits' partials are loaded in two halves.
__device__ void combine_rows(const PersistParams &p, int nsplit, int c, int ncta, int C, int tid) {
  const int sub = tid >> 6, d0 = (tid & 63) * 4;
  for (int base = c * 4; base < NH * C; base += ncta * 4) {
    const int row = base + sub;
    if (row >= NH * C) continue;
    const int h = row / C, q = row % C;
    float4 ov[MAXSPLIT];
    float2 ml[MAXSPLIT];
#pragma unroll
    for (int i = 0; i < MAXSPLIT; ++i) {
      if (i < nsplit) {
        const size_t r = ((size_t)i * NH + h) * 64 + q;
        ml[i] = __ldcg(reinterpret_cast<const float2 *>(p.mlpart + r * 2));
        ov[i] = __ldcg(reinterpret_cast<const float4 *>(p.opart + r * HD + d0));
      } else {
        ml[i] = make_float2(-INFINITY, 0.f);
        ov[i] = make_float4(0, 0, 0, 0);
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int i = 0; i < MAXSPLIT; ++i) M = fmaxf(M, ml[i].x);
    const float ref = (M == -INFINITY) ? 0.f : M;
    float L = 0.f;
    float4 a = make_float4(0, 0, 0, 0);
#pragma unroll
    for (int i = 0; i < MAXSPLIT; ++i) {
      const float w = exp2f(ml[i].x - ref);
      L += w * ml[i].y;
      a.x += w * ov[i].x;
      a.y += w * ov[i].y;
      a.z += w * ov[i].z;
      a.w += w * ov[i].w;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    uint2 v;
    v.x = pack_bf16(a.x * inv, a.y * inv);
    v.y = pack_bf16(a.z * inv, a.w * inv);
    *reinterpret_cast<uint2 *>(p.o + (size_t)q * 2048 + h * HD + d0) = v;
  }
}

// L2 prefetch of the table slices this CTA's units of GEMM phase gp will read: the operand
// scale or GELU bias slice, and the residual gate of the epilogue.  The weight producer issues
// it one phase ahead, so these small per-(step, layer) reads do not wait on HBM.
__device__ void prefetch_tables(const PersistParams &p, int gp, int c, int ncta) {
  if (gp >= p.S * p.L * 4) return;
  const int kind = gp & 3;
  const size_t kl = (size_t)(gp >> 2);
  for (int u = first_unit(gp, c, ncta); u < units(kind); u += ncta) {
    int nt, kb0, kb1;
    unit_kb(kind, u, nt, kb0, kb1);
    const uint32_t bytes = (uint32_t)(kb1 - kb0) * 64 * 4;
    if (kind == QKV) {
      bulk_prefetch_l2(p.s1p_attn + kl * D + kb0 * 64, bytes);
    } else if (kind == GU) {
      bulk_prefetch_l2(p.s1p_ffn + kl * D + kb0 * 64, bytes);
    } else if (kind == DN) {
      bulk_prefetch_l2(p.bias_gu + kl * 2 * F + kb0 * 64, bytes);
      bulk_prefetch_l2(p.bias_gu + kl * 2 * F + F + kb0 * 64, bytes);
      bulk_prefetch_l2(p.gate_ffn + kl * D + nt * 128, 512);
    } else {
      bulk_prefetch_l2(p.gate_attn + kl * D + nt * 128, 512);
    }
  }
}

// ---------------------------------------------------------------------------------------

// π0 suffix, token row c (CTA c, 256 threads): row 0 (the state token) gets W_st s + b_st in h;
// an action row gets the operand of the action-time output linear,
// op[c] = bf16(SiLU(W_fold x + c_k)), x = this row's actions (xr, 32 floats in shared memory).
// Thread t computes outputs t, t + 256, t + 512, t + 768, every weight load issued up front.
__device__ void pi0_row_in(const PersistParams &p, int c, int k, const float *xr, int tid) {
  float xv[A];
#pragma unroll
  for (int j = 0; j < A; ++j) xv[j] = xr[j];
#pragma unroll 1
  for (int e = 0; e < 4; ++e) {
    const int n = tid + NCOMP * e;
    if (c == 0) {
      uint4 w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) w[q] = __ldg(reinterpret_cast<const uint4 *>(p.w_st + (size_t)n * A) + q);
      float acc = __ldg(p.b_st + n);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bf16 *wb = reinterpret_cast<const bf16 *>(&w[q]);
#pragma unroll
        for (int t = 0; t < 8; ++t) acc += bf2f(wb[t]) * xv[q * 8 + t];
      }
      p.h[n] = acc;
    } else {
      float4 w[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) w[q] = __ldg(reinterpret_cast<const float4 *>(p.w_fold + (size_t)n * A) + q);
      float acc = __ldg(p.c_tab + (size_t)k * D + n);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        acc += w[q].x * xv[4 * q] + w[q].y * xv[4 * q + 1] + w[q].z * xv[4 * q + 2] + w[q].w * xv[4 * q + 3];
      p.op_ato[(size_t)c * D + n] = f2bf(acc / (1.0f + __expf(-acc)));
    }
  }
}

// π0: h[r][n] = b_ato[n] + sum_j op[r][j] W_ato[n][j] for the action rows r = 1 .. M-1.  CTA
// c < 64 takes output features 16c .. 16c + 15, two per warp.  The operand rows are staged in
// shared memory with a 16-byte pad per row (so that the lanes' rows fall in different banks);
// lane l accumulates rows 1 + l and 33 + l over the whole K, the weights read as broadcasts.
constexpr int OPS_LD = D / 8 + 1;  // staged operand row stride, in 16-byte chunks
__device__ void pi0_ato(const PersistParams &p, const Smem &sm, int c, int M, int tid) {
  if (c >= D / 16) return;
  uint4 *ops = reinterpret_cast<uint4 *>(sm.op);  // [64][OPS_LD] chunks of 8 bf16 (~129 KB)
  for (int i = tid; i < M * (D / 8); i += NCOMP)
    ops[(i >> 7) * OPS_LD + (i & 127)] = __ldcg(reinterpret_cast<const uint4 *>(p.op_ato) + i);
  named_sync();
  const int w = tid >> 5, lane = tid & 31;
  const int n0 = c * 16 + w * 2;
  const int ra = 1 + lane, rb = 33 + lane;
  const bool va = ra < M, vb = rb < M;
  const uint4 *oa = ops + (size_t)(va ? ra : 0) * OPS_LD, *ob = ops + (size_t)(vb ? rb : 0) * OPS_LD;
  const uint4 *w0 = reinterpret_cast<const uint4 *>(p.w_ato + (size_t)n0 * D);
  const uint4 *w1 = reinterpret_cast<const uint4 *>(p.w_ato + (size_t)(n0 + 1) * D);
  float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll 4
  for (int q = 0; q < D / 8; ++q) {
    const uint4 x0 = __ldg(w0 + q), x1 = __ldg(w1 + q), ya = oa[q], yb = ob[q];
    const bf16 *e0 = reinterpret_cast<const bf16 *>(&x0), *e1 = reinterpret_cast<const bf16 *>(&x1);
    const bf16 *fa = reinterpret_cast<const bf16 *>(&ya), *fb = reinterpret_cast<const bf16 *>(&yb);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const float u0 = bf2f(e0[t]), u1 = bf2f(e1[t]), ga = bf2f(fa[t]), gb = bf2f(fb[t]);
      a0 += u0 * ga;
      a1 += u1 * ga;
      b0 += u0 * gb;
      b1 += u1 * gb;
    }
  }
  const float bias0 = __ldg(p.b_ato + n0), bias1 = __ldg(p.b_ato + n0 + 1);
  if (va) {
    p.h[(size_t)ra * D + n0] = a0 + bias0;
    p.h[(size_t)ra * D + n0 + 1] = a1 + bias1;
  }
  if (vb) {
    p.h[(size_t)rb * D + n0] = b0 + bias0;
    p.h[(size_t)rb * D + n0 + 1] = b1 + bias1;
  }
}

__global__ void __launch_bounds__(THREADS, 1)
    k_persistent(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_o,
                 const __grid_constant__ CUtensorMap tm_gu, const __grid_constant__ CUtensorMap tm_d,
                 const __grid_constant__ CUtensorMap tm_rq, const __grid_constant__ CUtensorMap tm_rg,
                 const __grid_constant__ CUtensorMap tm_rh, const __grid_constant__ CUtensorMap tm_lh,
                 const __grid_constant__ CUtensorMap tm_lg, const __grid_constant__ CUtensorMap tm_lo,
                 const __grid_constant__ CUtensorMap tm_lq, const __grid_constant__ CUtensorMap tm_kc,
                 const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_ks,
                 const __grid_constant__ CUtensorMap tm_vs, PersistParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem sm;
  sm.ring = smem;
  sm.op = smem + RING * WST;
  sm.stg = sm.op + OPB;
  sm.tbl = reinterpret_cast<float *>(sm.stg + NGRP * GRPB);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm.op + REGION);
  sm.full = bars;
  sm.empty = bars + RING;
  sm.opf = bars + 2 * RING;
  sm.stgb = sm.opf + NOPK;
  sm.acc_ready = sm.stgb + NGRP;
  sm.drain = sm.acc_ready + 1;
  sm.att = sm.drain + 1;
  sm.tblb = sm.att + 1;
  sm.tmem_slot = reinterpret_cast<uint32_t *>(sm.tblb + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x, ncta = gridDim.x;
  const int L = p.L, S = p.S;
  DevCtl *ctl = p.ctl;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBARS; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_o);
    tma_prefetch_desc(&tm_gu);
    tma_prefetch_desc(&tm_d);
  }
  if (warp == 1) {
    tmem_alloc(sm.tmem_slot, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ weight producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      uint32_t it = 0;
      bool ok = true;
      for (int k = 0; k < S && ok; ++k)
        for (int l = 0; l < L && ok; ++l)
          for (int kind = 0; kind < 4 && ok; ++kind) {
            const int gp = (k * L + l) * 4 + kind;
            prefetch_tables(p, gp + 1, c, ncta);
            for (int u = first_unit(gp, c, ncta); u < units(kind) && ok; u += ncta) {
              int nt, kb0, kb1;
              unit_kb(kind, u, nt, kb0, kb1);
              for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int slot = it % RING;
                if (it >= RING && !wait_bar(&sm.empty[slot], ((it / RING) & 1) ^ 1, ctl, 611)) {
                  ok = false;
                  break;
                }
                const CUtensorMap *map =
                    kind == QKV ? &tm_qkv : (kind == OPJ ? &tm_o : (kind == GU ? &tm_gu : &tm_d));
                mbar_arrive_expect_tx(&sm.full[slot], WST);
                tma_load_2d(sm.ring + slot * WST, map, &sm.full[slot], kb * 64, l * rows_per_layer(kind) + nt * 128,
                            pol);
              }
            }
          }
      // every issued copy must land before the CTA may exit
      const uint32_t first = it > (uint32_t)RING ? it - RING : 0;
      for (uint32_t j = first; j < it; ++j) wait_bar(&sm.full[j % RING], (j / RING) & 1, ctl, 612, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, 64);
      const uint32_t opb = smem_u32(sm.op);
      uint32_t it = 0, opf_par = 0;
      bool ok = true;
      for (int k = 0; k < S && ok; ++k)
        for (int l = 0; l < L && ok; ++l)
          for (int kind = 0; kind < 4 && ok; ++kind) {
            const int gp = (k * L + l) * 4 + kind;
            for (int u = first_unit(gp, c, ncta); u < units(kind) && ok; u += ncta) {
              int nt, kb0, kb1;
              unit_kb(kind, u, nt, kb0, kb1);
              for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int j = kb - kb0;
                if (!wait_bar(&sm.opf[j], (opf_par >> j) & 1, ctl, 621)) {
                  ok = false;
                  break;
                }
                opf_par ^= 1u << j;
                const int slot = it % RING;
                if (!wait_bar(&sm.full[slot], (it / RING) & 1, ctl, 622)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
                const uint32_t a = smem_u32(sm.ring + slot * WST);
                const uint32_t b = opb + j * 8192;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  umma_bf16(tmem, sdesc_k128(a + 32 * q), sdesc_k128(b + 32 * q), idesc,
                            (kb > kb0 || q > 0) ? 1u : 0u);
                umma_commit(&sm.empty[slot]);
              }
              if (ok) umma_commit(sm.acc_ready);
            }
          }
      umma_commit(sm.drain);
      wait_bar(sm.drain, 0, ctl, 623, false);
    }
  } else {
    // ------------------------------------------------------------------ compute warps
    const int tid = threadIdx.x - 64;
    const int cw = warp - 2;
    const int C = p.C, M = p.C;
    unsigned epoch = 0;
    uint32_t nunit = 0, gstg = 0, natt = 0, ntbl = 0;
    const CallArgs *ca = p.ca;
    AttnCtx ac;
    ac.lv = ca->valid_len[0];
    if (ac.lv < 0 || ac.lv > p.ca_cap) {
      if (tid == 0 && c == 0) set_error(ctl, DEVERR_BOUNDS, 631);
      ac.lv = ac.lv < 0 ? 0 : p.ca_cap;
    }
    ac.npre = (ac.lv + KC - 1) / KC;
    ac.nsuf = (C + KC - 1) / KC;
    ac.cps = p.attn_cps;
    ac.nsplit = p.attn_splits;

    // ---- init: x = noise, h = action_in(x); zero the accumulators and the unused rows
    zero_slice(p.acc_qkv, (size_t)64 * 2560, c, ncta, tid);
    zero_slice(p.acc_gu, (size_t)64 * 2 * F, c, ncta, tid);
    if (c == 0)
      for (int i = tid; i < 128; i += NCOMP) (i < 64 ? p.ss_attn : p.ss_ffn)[i & 63] = 0.f;
    for (int i = c * NCOMP + tid; i < (64 - C) * 2048; i += ncta * NCOMP) {
      p.o[(size_t)C * 2048 + i] = f2bf(0.f);
      p.qb[(size_t)C * 2048 + i] = f2bf(0.f);
    }
    float *xs = reinterpret_cast<float *>(sm.op);
    if (p.pi0 && c < M) {
      // π0: the state row, and the action rows' operands of the action-time output linear
      if (tid < A) {
        float v;
        if (c == 0) {
          v = ca->state[tid];
        } else {
          v = ca->noise[(c - 1) * A + tid];
          p.x[c * A + tid] = v;
        }
        xs[tid] = v;
      }
      named_sync();
      pi0_row_in(p, c, 0, xs, tid);
    } else if (c < M) {
      if (tid < A) {
        const float v = ca->noise[c * A + tid];
        p.x[c * A + tid] = v;
        xs[tid] = v;
      }
      named_sync();
      for (int n = tid; n < D; n += NCOMP) {
        float a = p.b_in[n];
        for (int j = 0; j < A; ++j) a += bf2f(p.w_in[n * A + j]) * xs[j];
        p.h[(size_t)c * D + n] = a;
      }
    } else if (c < 64) {
      for (int n = tid; n < D; n += NCOMP) p.h[(size_t)c * D + n] = 0.f;
    }
    grid_sync(p, p.bar, ctl, epoch, ncta, tid);
    if (p.pi0) {
      pi0_ato(p, sm, c, M, tid);
      grid_sync(p, p.bar, ctl, epoch, ncta, tid);
    }

    for (int k = 0; k < S; ++k) {
      for (int l = 0; l < L; ++l) {
        const size_t kl = (size_t)k * L + l;
        for (int kind = 0; kind < 4; ++kind) {
          if (kind == OPJ) {
            // ---- finalise Q/K/V (bf16, RoPE) once, then attention, then the split merge
            if (c == 0)
              for (int i = tid; i < 64; i += NCOMP) p.ss_ffn[i] = 0.f;
            zero_slice(p.acc_gu, (size_t)M * 2 * F, c, ncta, tid);
            qkv_finalise(p, ac.lv, kl, c, ncta, C, tid);
            grid_sync(p, p.bar, ctl, epoch, ncta, tid);
            zero_slice(p.acc_qkv, (size_t)M * 2560, c, ncta, tid);
            for (int u = c; u < NH * ac.nsplit; u += ncta)
              attn_unit(p, sm, ac, u % NH, u / NH, l, &tm_lq, &tm_kc, &tm_vc, &tm_ks, &tm_vs, natt, tid, epoch);
            grid_sync(p, p.bar, ctl, epoch, ncta, tid);
            combine_rows(p, ac.nsplit, c, ncta, C, tid);
            if (c == 0)
              for (int i = tid; i < 64; i += NCOMP) p.ss_attn[i] = 0.f;
            grid_sync(p, p.bar, ctl, epoch, ncta, tid);
          }
          if (kind == QKV && p.trace != nullptr && k == p.trace_step) {
            // test trace: the layer's input h (complete since the last barrier; this phase
            // only reads it)
            float *dst = p.trace + (size_t)l * C * D;
            for (int i = (c * NCOMP + tid) * 4; i < C * D; i += ncta * NCOMP * 4)
              *reinterpret_cast<float4 *>(dst + i) = __ldcg(reinterpret_cast<const float4 *>(p.h + i));
          }
          const int gp = (int)kl * 4 + kind;
          for (int u = first_unit(gp, c, ncta); u < units(kind); u += ncta, ++nunit) {
            int nt, kb0, kb1;
            unit_kb(kind, u, nt, kb0, kb1);
            const int nkb = kb1 - kb0;
            if (kind == OPJ) {
              // the attention output is already bf16: TMA it straight into the operand
              if (tid == 0) {
                const uint64_t pol = policy_evict_last();
                for (int j = 0; j < nkb; ++j) {
                  mbar_arrive_expect_tx(&sm.opf[j], 8192);
                  tma_load_2d(sm.op + j * 8192, &tm_lo, &sm.opf[j], (kb0 + j) * 64, 0, pol);
                }
              }
            } else if (kind == QKV) {
              build_operand(p, sm, &tm_lh, &tm_lg, kind, kb0, nkb, p.s1p_attn + kl * D, nullptr, p.ss_attn, nt == 0,
                            M, gstg, ntbl, tid);
            } else if (kind == GU) {
              build_operand(p, sm, &tm_lh, &tm_lg, kind, kb0, nkb, p.s1p_ffn + kl * D, nullptr, p.ss_ffn, nt == 0, M,
                            gstg, ntbl, tid);
            } else {
              build_operand(p, sm, &tm_lh, &tm_lg, kind, kb0, nkb, nullptr, p.bias_gu + kl * 2 * F, p.ss_ffn, false,
                            M, gstg, ntbl, tid);
            }
            if (tid == 0) stamp(p, epoch, 1);
            // epilogue: TMEM -> registers (x gate) -> shared tile [64 tokens][128 features] ->
            // one TMA bulk reduce-add into the fp32 destination
            float *tile = reinterpret_cast<float *>(sm.op);
            const int q = warp & 3, half = cw >> 2;
            const int nl = q * 32 + lane;
            float sc = 1.f;  // AdaRMS gate of the residual, loaded before the accumulator is ready
            if (kind == OPJ || kind == DN) sc = __ldg((kind == OPJ ? p.gate_attn : p.gate_ffn) + kl * D + nt * 128 + nl);
            if (wait_bar(sm.acc_ready, nunit & 1, ctl, 632)) {
              tc_fence_after();
              if (tid == 0) stamp(p, epoch, 2);
              float v[32];
              tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * 32), v);
#pragma unroll
              for (int j = 0; j < 32; ++j) tile[(half * 32 + j) * 128 + nl] = v[j] * sc;
            }
            tc_fence_before();
            fence_proxy_async_shared();
            named_sync();
            if (tid == 0) {
              const CUtensorMap *dst = kind == QKV ? &tm_rq : (kind == GU ? &tm_rg : &tm_rh);
              tma_reduce_add_2d(dst, tile, nt * 128, 0);
              bulk_commit();
              // a later unit of this phase reuses the tile; the last one is covered by the barrier
              if (u + ncta < units(kind)) bulk_wait_read0();
              stamp(p, epoch, 3);
            }
            named_sync();
          }
          grid_sync(p, p.bar, ctl, epoch, ncta, tid);
        }
      }
      // ---- final AdaRMS + action_out_proj (dt folded) + Euler; next step's action_in.
      // CTA c < M owns token row c; thread t owns elements 4t..4t+3 of it.
      if (p.pi0 && c == 0) {
        // π0 state row: no action of its own; the next step restarts it from the state
        if (p.trace != nullptr && k == p.trace_step) {
          const int n0 = tid * 4;
          *reinterpret_cast<float4 *>(p.trace + (size_t)L * C * D + n0) =
              __ldcg(reinterpret_cast<const float4 *>(p.h + n0));
        }
        if (k < S - 1) {
          float *xr = reinterpret_cast<float *>(sm.op);
          if (tid < A) xr[tid] = ca->state[tid];
          named_sync();
          pi0_row_in(p, 0, k + 1, xr, tid);
        }
      } else if (c < M) {
        float *red = reinterpret_cast<float *>(sm.op);  // [8 warps][33]
        float *xr = red + 8 * 33;
        const int n0 = tid * 4;
        const float4 hv = __ldcg(reinterpret_cast<const float4 *>(p.h + (size_t)c * D + n0));
        if (p.trace != nullptr && k == p.trace_step)
          *reinterpret_cast<float4 *>(p.trace + ((size_t)L * C + c) * D + n0) = hv;
        float ss = hv.x * hv.x + hv.y * hv.y + hv.z * hv.z + hv.w * hv.w;
        ss = warp_sum(ss);
        if (lane == 0) red[cw * 33 + 32] = ss;
        named_sync();
        float tot = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) tot += red[i * 33 + 32];
        const float r = rsqrtf(tot * (1.0f / D) + p.eps);
        float nv[4] = {hv.x, hv.y, hv.z, hv.w};
        if (p.final_norm) {
          const float4 sc = __ldg(reinterpret_cast<const float4 *>(p.s1p_fin + (size_t)k * D + n0));
          const float4 sh = __ldg(reinterpret_cast<const float4 *>(p.shift_fin + (size_t)k * D + n0));
          nv[0] = r * hv.x * sc.x + sh.x;
          nv[1] = r * hv.y * sc.y + sh.y;
          nv[2] = r * hv.z * sc.z + sh.z;
          nv[3] = r * hv.w * sc.w + sh.w;
        }
        float part[A];
#pragma unroll
        for (int hb = 0; hb < 4; ++hb) {
          float4 w[8];
#pragma unroll
          for (int a = 0; a < 8; ++a)
            w[a] = __ldg(reinterpret_cast<const float4 *>(p.w_out + (size_t)(hb * 8 + a) * D + n0));
#pragma unroll
          for (int a = 0; a < 8; ++a)
            part[hb * 8 + a] = nv[0] * w[a].x + nv[1] * w[a].y + nv[2] * w[a].z + nv[3] * w[a].w;
        }
#pragma unroll
        for (int a = 0; a < A; ++a) {
          const float v = warp_sum(part[a]);
          if (lane == a) red[cw * 33 + a] = v;
        }
        named_sync();
        if (tid < A) {
          float v = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) v += red[i * 33 + tid];
          const float nx = __ldcg(p.x + c * A + tid) + v + __ldg(p.b_out + tid);
          p.x[c * A + tid] = nx;
          xr[tid] = nx;
          if (k == S - 1 && ca->actions != nullptr) ca->actions[(c - p.pi0) * A + tid] = nx;
        }
        named_sync();
        if (k < S - 1 && p.pi0) {
          pi0_row_in(p, c, k + 1, xr, tid);
        } else if (k < S - 1) {
          uint4 wi[4][4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              wi[e][j] = __ldg(reinterpret_cast<const uint4 *>(p.w_in + (size_t)(n0 + e) * A + j * 8));
          float4 out;
          float *ov = reinterpret_cast<float *>(&out);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float a = __ldg(p.b_in + n0 + e);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const bf16 *wb = reinterpret_cast<const bf16 *>(&wi[e][j]);
#pragma unroll
              for (int q = 0; q < 8; ++q) a += bf2f(wb[q]) * xr[j * 8 + q];
            }
            ov[e] = a;
          }
          *reinterpret_cast<float4 *>(p.h + (size_t)c * D + n0) = out;
        }
      }
      if (k < S - 1) grid_sync(p, p.bar, ctl, epoch, ncta, tid);
      if (k < S - 1 && p.pi0) {
        pi0_ato(p, sm, c, M, tid);
        grid_sync(p, p.bar, ctl, epoch, ncta, tid);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

}  // namespace pk

int persistent_max_splits(int sm_count) {
  return sm_count / pk::NH < pk::MAXSPLIT ? sm_count / pk::NH : pk::MAXSPLIT;
}

int persistent_smem_bytes() { return pk::SMEM; }

cudaError_t persistent_init_attributes() {
  return cudaFuncSetAttribute(pk::k_persistent, cudaFuncAttributeMaxDynamicSharedMemorySize, pk::SMEM);
}

bool persistent_fits(int sm_count) {
  int blocks = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, pk::k_persistent, pk::THREADS, pk::SMEM) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return blocks >= 1 && sm_count >= 64;
}

void persistent_attn_plan(int cap, int chunk, int sm_count, int *splits, int *cps) {
  const int chunks = (cap + pk::KC - 1) / pk::KC + (chunk + pk::KC - 1) / pk::KC;
  int s = persistent_max_splits(sm_count);
  if (s > chunks) s = chunks;
  if (s < 1) s = 1;
  *cps = (chunks + s - 1) / s;
  *splits = (chunks + *cps - 1) / *cps;
}

cudaError_t persistent_launch(const PersistMaps &m, const PersistParams &p, int grid, cudaStream_t st) {
  void *args[] = {const_cast<CUtensorMap *>(&m.w_qkv), const_cast<CUtensorMap *>(&m.w_o),
                  const_cast<CUtensorMap *>(&m.w_gu),  const_cast<CUtensorMap *>(&m.w_d),
                  const_cast<CUtensorMap *>(&m.r_qkv), const_cast<CUtensorMap *>(&m.r_gu),
                  const_cast<CUtensorMap *>(&m.r_h),   const_cast<CUtensorMap *>(&m.l_h),
                  const_cast<CUtensorMap *>(&m.l_gu),  const_cast<CUtensorMap *>(&m.l_o),
                  const_cast<CUtensorMap *>(&m.l_q),   const_cast<CUtensorMap *>(&m.l_kc),
                  const_cast<CUtensorMap *>(&m.l_vc),  const_cast<CUtensorMap *>(&m.l_ks),
                  const_cast<CUtensorMap *>(&m.l_vs),  const_cast<PersistParams *>(&p)};
  return cudaLaunchCooperativeKernel(reinterpret_cast<void *>(pk::k_persistent), dim3(grid), dim3(pk::THREADS), args,
                                     pk::SMEM, st);
}

}  // namespace rtvla
