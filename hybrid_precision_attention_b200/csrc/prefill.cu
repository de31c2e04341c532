// prefill.cu — hybrid-precision causal prefill attention on tcgen05 tensor cores.
//
// HyQuant digest (agihunt.info), prefill/decode paragraph; repository README,
// Overview item 2 and the "vquant_vert" / "hybrid_full" modes: in prefill the
// quantised path and the full-precision path are fused into one
// FlashAttention-style kernel; most of the attention GEMM work runs in low
// precision while the vertical-line and local-window tiles stay FP16/BF16, and
// one online softmax covers both.  The pages' kernels are Triton (FP8 on SM90);
// this is a B200 design.
//
// What is computed, for query i and key j <= i of (b, head):
//   window key  (i - W < j <= i)            : FP16 Q, K, V
//   VL key      (j in the vertical-line set) : FP16 Q, K, V
//   other key                                : FP8 e4m3 Q, K, V, one float32 scale per
//                                              (b, head, 128 positions): x8 = e4m3(x / s)
// then one softmax over all of them.  A vertical line inside the window counts
// once, as a window key.
//
// Kernels
//   fp8_block_quant  per (b, head, 128-position block): amax, scale = amax/448,
//                    e4m3 codes (Q, K) or the e4m3 value times the scale stored as
//                    fp16 (V, so that P.V runs on the f16 tensor path with no
//                    per-key scale); rows past L are zero
//   kbias_init       score bias of the e4m3 key blocks: 0, or -inf past L
//   vl_prep          -inf bias on the vertical lines and the VL rows of K and V
//                    gathered into contiguous 128-row tiles (positions padded with
//                    INT_MAX)
//   prefill_kernel   one CTA per (128-query tile, query head, batch):
//                      warps 0-3  softmax, one query row per thread = one TMEM lane
//                      warp 4     TMA producers: lane 0 Q once and the K tiles (with
//                                 their score bias or VL positions and K scales),
//                                 lane 1 the V tiles; 2 stages each
//                      warp 5     TMEM allocation and the tcgen05.mma issue
//                    key tiles in order: FP8 tiles (QK on kind::f8f6f4), VL tiles
//                    and window tiles (QK on kind::f16); S = Q K^T lands in one of
//                    two TMEM buffers, the softmax reads it, writes P (fp16) to
//                    shared memory in the 128-byte-swizzled K-major layout, and
//                    O += P V (kind::f16, V MN-major) accumulates in TMEM.  QK runs
//                    two tiles ahead of the softmax; a K stage is free once its QK
//                    is done, a V stage once its PV is.  The running max is
//                    refreshed lazily (O in TMEM is rescaled only when the max
//                    grows by more than 2^8).
// All mbarrier waits are bounded (about 1 s); a timeout sets the error word and
// the CTA drains its copies and MMAs before releasing TMEM.
#include <climits>
#include <cstdio>
#include <cuda_fp8.h>

#include "tc.cuh"

namespace hq {
namespace {

constexpr int TQ = 128, TKEY = 128;
constexpr int PF_THREADS = 192;
constexpr float E4M3_MAX = 448.0f;
// shared memory map (byte offsets from a 1024-byte aligned base)
constexpr int SM_Q8 = 0;                        // Q e4m3   [128][128 B]            16 KB
constexpr int SM_Q16 = 16384;                   // Q fp16   2 x [128][128 B]        32 KB
constexpr int SM_K = 49152;                     // 2 K stages x 32 KB (e4m3 tiles use the first 16 KB)
constexpr int SM_V = SM_K + 2 * 32768;          // 2 V stages x 32 KB (fp16, 2 x [128 keys][128 B])
constexpr int SM_P = SM_V + 2 * 32768;          // P fp16   2 x [128][128 B]        32 KB
constexpr int SM_AUX = SM_P + 32768;            // 2 K stages x 1 KB: [0,512) mask bias or VL positions, [512,528) K scales
constexpr int AUX_STAGE = 1024;
constexpr int SM_USED = SM_AUX + 2 * AUX_STAGE;
constexpr int PF_SMEM = SM_USED + 1024;         // + slack for the 1024-byte alignment
constexpr uint32_t TMEM_COLS = 512;             // S double buffer: columns 0..255, O: 256..383
constexpr uint32_t TM_O = 256;
constexpr uint32_t IDESC_QK = idesc_make(0, 0, 0, TQ, TKEY);   // K-major A and B
constexpr uint32_t IDESC_PV = idesc_make(0, 0, 1, TQ, 128);    // A = P K-major, B = V MN-major

struct Tmaps {
  CUtensorMap q8, q16, k8, v8, k16, v16, kvl, vvl;
};

struct PfArgs {
  int B, Hq, Hkv, L, Lp, nblk, W, n_vl, nvlp;
  float qk_scale;        // sm_scale * log2(e)
  const float* sq;       // [B*Hq][nblk]
  const float* sk;       // [B*Hkv][nblk] (16-byte readable past the end)
  const float* kbias;    // [B*Hkv][Lp]: -inf on vertical lines and past L, else 0
  const int32_t* vlpos;  // [B*Hkv][nvlp], INT_MAX padded
  uint16_t* out;         // [B, Hq, L, D]
  uint32_t* err;         // device error word
};

__device__ __forceinline__ bool waitb(uint64_t* bar, uint32_t parity, uint32_t* err, int* abort_flag) {
  if (*reinterpret_cast<volatile int*>(abort_flag)) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile int*>(abort_flag)) return false;
    if (global_ns() - t0 > 1000000000ull) {
      atomicOr(err, 1u);
      *reinterpret_cast<volatile int*>(abort_flag) = 1;
      return false;
    }
  }
}

// per-CTA tile schedule
struct Sched {
  int qt, q0, imax, nA, nB, nC, ktw0, nvv, nT;
};

__device__ __forceinline__ int count_le(const int32_t* a, int n, int key) {
  int lo = 0, hi = n;  // number of a[0..n) <= key (ascending)
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] <= key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ Sched schedule(const PfArgs& a, int bk) {
  Sched s;
  s.qt = gridDim.x - 1 - blockIdx.x;  // longest rows first
  s.q0 = s.qt * TQ;
  s.imax = min(s.q0 + TQ - 1, a.L - 1);
  const int jmax = s.imax - a.W;  // largest key any row of the tile sees outside its window
  s.nA = jmax >= 0 ? jmax / TKEY + 1 : 0;
  s.nvv = jmax >= 0 ? count_le(a.vlpos + static_cast<size_t>(bk) * a.nvlp, a.n_vl, jmax) : 0;
  s.nB = (s.nvv + TKEY - 1) / TKEY;
  if (a.W > 0) {
    const int wlo = max(0, s.q0 - a.W + 1);
    s.ktw0 = wlo / TKEY;
    s.nC = s.imax / TKEY - s.ktw0 + 1;
  } else {
    s.ktw0 = 0;
    s.nC = 0;
  }
  s.nT = s.nA + s.nB + s.nC;
  return s;
}

// Tiles t of a CTA in order: [0, nA) e4m3 key blocks 0 .. nA-1, [nA, nA+nB) VL
// tiles, then the window's fp16 key blocks from ktw0.  Pipeline (all waits bounded):
//   K lane   K(t) -> K stage t%2 (+ mask bias / VL positions and the K scales)
//   V lane   V(t) -> V stage t%2
//   MMA      QK(t) -> S buffer t%2 (two tiles ahead of the softmax), PV(t) -> O
//   softmax  S(t) -> P (fp16, shared memory) -> PV(t)
__global__ void __launch_bounds__(PF_THREADS, 1) prefill_kernel(const __grid_constant__ Tmaps tm, const PfArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t q_full, p_full, o_done, drain, k_full[2], k_empty[2], v_full[2], v_empty[2],
      s_full[2], s_free[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int hq = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  const int kvh = hq / G;
  const int bq = b * a.Hq + hq, bk = b * a.Hkv + kvh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Sched sc = schedule(a, bk);

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&p_full, 128);
    mbar_init(&o_done, 1);
    mbar_init(&drain, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t sm_base = smem_u32(sm);

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producers
    // lane 0: Q once, then the K tiles with their auxiliary data; lane 1: the V
    // tiles.  The two lanes wait on different barriers independently.
    if (lane == 0) {
      mbar_arrive_expect_tx(&q_full, 16384 + 32768);
      tma_load_3d(sm + SM_Q8, &tm.q8, 0, sc.q0, bq, &q_full);
      tma_load_3d(sm + SM_Q16, &tm.q16, 0, sc.q0, bq, &q_full);
      tma_load_3d(sm + SM_Q16 + 16384, &tm.q16, 64, sc.q0, bq, &q_full);
      int issued[2] = {0, 0};
      for (int t = 0; t < sc.nT; ++t) {
        const int s = t & 1;
        // the stage is free once QK(t-2) is done and the softmax has read the
        // stage's mask bias / VL positions / K scales of tile t-2
        if (t >= 2 && !(waitb(&k_empty[s], ((t >> 1) - 1) & 1, a.err, &abort_flag) &&
                        waitb(&s_free[s], ((t >> 1) - 1) & 1, a.err, &abort_flag)))
          break;
        uint8_t* K = sm + SM_K + s * 32768;
        uint8_t* aux = sm + SM_AUX + s * AUX_STAGE;
        if (t < sc.nA) {
          const int kt = t;
          mbar_arrive_expect_tx(&k_full[s], 16384 + 512 + 16);
          tma_load_3d(K, &tm.k8, 0, kt * TKEY, bk, &k_full[s]);
          bulk_g2s(aux, a.kbias + static_cast<size_t>(bk) * a.Lp + kt * TKEY, 512, &k_full[s]);
          bulk_g2s(aux + 512, a.sk + ((static_cast<size_t>(bk) * a.nblk + kt) & ~static_cast<size_t>(3)), 16, &k_full[s]);
        } else if (t < sc.nA + sc.nB) {
          const int v = t - sc.nA;
          mbar_arrive_expect_tx(&k_full[s], 32768 + 512);
          tma_load_3d(K, &tm.kvl, 0, v * TKEY, bk, &k_full[s]);
          tma_load_3d(K + 16384, &tm.kvl, 64, v * TKEY, bk, &k_full[s]);
          bulk_g2s(aux, a.vlpos + static_cast<size_t>(bk) * a.nvlp + v * TKEY, 512, &k_full[s]);
        } else {
          const int kt = sc.ktw0 + (t - sc.nA - sc.nB);
          mbar_arrive_expect_tx(&k_full[s], 32768);
          tma_load_3d(K, &tm.k16, 0, kt * TKEY, bk, &k_full[s]);
          tma_load_3d(K + 16384, &tm.k16, 64, kt * TKEY, bk, &k_full[s]);
        }
        issued[s] = (t >> 1) + 1;
      }
      if (abort_flag) {
        // never expected: let every issued copy land before the CTA can exit
        int dummy = 0;
        for (int s = 0; s < 2; ++s)
          if (issued[s] > 0) waitb(&k_full[s], (issued[s] - 1) & 1, a.err, &dummy);
        waitb(&q_full, 0, a.err, &dummy);
      }
    } else if (lane == 1) {
      int issued[2] = {0, 0};
      for (int t = 0; t < sc.nT; ++t) {
        const int s = t & 1;
        if (t >= 2 && !waitb(&v_empty[s], ((t >> 1) - 1) & 1, a.err, &abort_flag)) break;
        uint8_t* V = sm + SM_V + s * 32768;
        const CUtensorMap* map;
        int row;
        if (t < sc.nA) {
          map = &tm.v8;
          row = t * TKEY;
        } else if (t < sc.nA + sc.nB) {
          map = &tm.vvl;
          row = (t - sc.nA) * TKEY;
        } else {
          map = &tm.v16;
          row = (sc.ktw0 + (t - sc.nA - sc.nB)) * TKEY;
        }
        mbar_arrive_expect_tx(&v_full[s], 32768);
        tma_load_3d(V, map, 0, row, bk, &v_full[s]);
        tma_load_3d(V + 16384, map, 64, row, bk, &v_full[s]);
        issued[s] = (t >> 1) + 1;
      }
      if (abort_flag) {
        int dummy = 0;
        for (int s = 0; s < 2; ++s)
          if (issued[s] > 0) waitb(&v_full[s], (issued[s] - 1) & 1, a.err, &dummy);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t q8 = sm_base + SM_Q8, q16 = sm_base + SM_Q16, p = sm_base + SM_P;
      bool ok = waitb(&q_full, 0, a.err, &abort_flag);
      // QK(t) into S buffer t%2, once K(t) landed and the softmax has read S(t-2)
      auto issue_qk = [&](int t) -> bool {
        const int s = t & 1;
        if (!waitb(&k_full[s], (t >> 1) & 1, a.err, &abort_flag)) return false;
        if (t >= 2 && !waitb(&s_free[s], ((t >> 1) - 1) & 1, a.err, &abort_flag)) return false;
        tc_fence_after();
        const uint32_t S = tmem + 128 * s;
        const uint32_t K = sm_base + SM_K + s * 32768;
        if (t < sc.nA) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f8(S, sdesc_sw128(q8 + 32 * kk, 16, 1024), sdesc_sw128(K + 32 * kk, 16, 1024), IDESC_QK, kk > 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + 32 * (kk & 3);
            umma_f16(S, sdesc_sw128(q16 + off, 16, 1024), sdesc_sw128(K + off, 16, 1024), IDESC_QK, kk > 0);
          }
        }
        umma_commit(&s_full[s]);
        umma_commit(&k_empty[s]);
        return true;
      };
      if (ok && sc.nT > 0) ok = issue_qk(0);
      if (ok && sc.nT > 1) ok = issue_qk(1);
      for (int t = 0; ok && t < sc.nT; ++t) {
        const int s = t & 1;
        ok = waitb(&p_full, t & 1, a.err, &abort_flag) && waitb(&v_full[s], (t >> 1) & 1, a.err, &abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t V = sm_base + SM_V + s * 32768;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * 16384 + 32 * (kk & 3);
          umma_f16(tmem + TM_O, sdesc_sw128(p + aoff, 16, 1024), sdesc_sw128(V + 2048 * kk, 16384, 1024), IDESC_PV,
                   (t > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&o_done);
        umma_commit(&v_empty[s]);
        if (t + 2 < sc.nT) ok = issue_qk(t + 2);
      }
      // every MMA this thread issued completes before TMEM is released
      umma_commit(&drain);
      int dummy = 0;
      waitb(&drain, 0, a.err, &dummy);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0..3)
    const int r = threadIdx.x;  // row within the tile = TMEM lane
    const int i = sc.q0 + r;
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const uint32_t prow = sm_base + SM_P + r * 128;
    float m_run = -INFINITY, l_run = 0.f;
    const float sqv = a.sq[static_cast<size_t>(bq) * a.nblk + sc.qt];
    bool ok = true;
    for (int t = 0; t < sc.nT; ++t) {
      const int s = t & 1;
      ok = ok && waitb(&s_full[s], (t >> 1) & 1, a.err, &abort_flag);
      if (!__all_sync(0xffffffffu, ok)) ok = false;
      if (!ok) break;
      tc_fence_after();
      float x[TKEY];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld32f(trow + 128 * s + 32 * c4, x + 32 * c4);
      tmem_wait_ld();

      // scale and mask this tile's scores
      const uint8_t* aux = sm + SM_AUX + s * AUX_STAGE;
      float mt = -INFINITY;
      if (t < sc.nA) {
        const int kt = t;
        const float skv = reinterpret_cast<const float*>(aux + 512)[(static_cast<size_t>(bk) * a.nblk + kt) & 3];
        const float scl = sqv * skv * a.qk_scale;
        const float4* bias = reinterpret_cast<const float4*>(aux);
        const int jlim = i - a.W - kt * TKEY;  // causal limit of this row: columns c <= jlim
        if (jlim >= TKEY - 1) {
#pragma unroll
          for (int c4 = 0; c4 < TKEY / 4; ++c4) {
            const float4 bb = bias[c4];
            x[4 * c4] = fmaf(x[4 * c4], scl, bb.x);
            x[4 * c4 + 1] = fmaf(x[4 * c4 + 1], scl, bb.y);
            x[4 * c4 + 2] = fmaf(x[4 * c4 + 2], scl, bb.z);
            x[4 * c4 + 3] = fmaf(x[4 * c4 + 3], scl, bb.w);
            mt = fmaxf(mt, fmaxf(fmaxf(x[4 * c4], x[4 * c4 + 1]), fmaxf(x[4 * c4 + 2], x[4 * c4 + 3])));
          }
        } else {
#pragma unroll
          for (int c4 = 0; c4 < TKEY / 4; ++c4) {
            const float4 bb = bias[c4];
            const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 4 * c4 + e;
              x[c] = c <= jlim ? fmaf(x[c], scl, bv[e]) : -INFINITY;
              mt = fmaxf(mt, x[c]);
            }
          }
        }
      } else if (t < sc.nA + sc.nB) {
        const int32_t* vp = reinterpret_cast<const int32_t*>(aux);
        const int lim = i - a.W;
#pragma unroll
        for (int c = 0; c < TKEY; ++c) {
          const bool v = vp[c] <= lim;
          x[c] = v ? x[c] * a.qk_scale : -INFINITY;
          mt = fmaxf(mt, x[c]);
        }
      } else {
        const int kt = sc.ktw0 + (t - sc.nA - sc.nB);
        const int lo = i - a.W + 1 - kt * TKEY, hi = i - kt * TKEY;  // window: lo <= c <= hi
#pragma unroll
        for (int c = 0; c < TKEY; ++c) {
          const bool v = c >= lo && c <= hi;
          x[c] = v ? x[c] * a.qk_scale : -INFINITY;
          mt = fmaxf(mt, x[c]);
        }
      }
      // S(t) is in registers and the stage's auxiliary data has been read: the S
      // buffer and the K stage's aux area may be refilled
      tc_fence_before();
      mbar_arrive(&s_free[s]);
      // lazy running max: only move it (and rescale O) when it grows by > 2^8
      const bool grow = mt > m_run + 8.0f;
      const bool any_grow = __any_sync(0xffffffffu, grow);
      float alpha = 1.f;
      if (grow) {
        alpha = m_run != -INFINITY ? ex2(m_run - mt) : 0.f;
        m_run = mt;
        l_run *= alpha;
      }
      // P = exp2(s - m_run) in fp16, row sum in fp32
      const float mref = m_run == -INFINITY ? 0.f : m_run;
      uint32_t pk[TKEY / 2];
      float l0 = 0.f, l1 = 0.f;
#pragma unroll
      for (int c = 0; c < TKEY; c += 2) {
        const float p0 = ex2(x[c] - mref), p1 = ex2(x[c + 1] - mref);
        l0 += p0;
        l1 += p1;
        pk[c / 2] = pack_f16x2(p0, p1);
      }
      l_run += l0 + l1;
      // O holds P.V of earlier tiles and the P buffer is read by PV of tile t-1:
      // wait for it, then (if the max moved) rescale O in TMEM
      if (t > 0) {
        ok = waitb(&o_done, (t - 1) & 1, a.err, &abort_flag);
        if (!__all_sync(0xffffffffu, ok)) ok = false;
        if (!ok) break;
        if (any_grow) {
          tc_fence_after();
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t u[32];
            tmem_ld32(trow + TM_O + 32 * c4, u);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
            tmem_st32(trow + TM_O + 32 * c4, u);
          }
          tmem_wait_st();
        }
      }
      // store P row r (K-major, 128-byte swizzle: 16-byte chunk k of the row goes
      // to chunk k ^ (r % 8) of the 128-byte line; keys 64..127 in region 1)
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const uint32_t addr = prow + (k >> 3) * 16384 + ((((k & 7) ^ (r & 7))) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * k]), "r"(pk[4 * k + 1]),
                     "r"(pk[4 * k + 2]), "r"(pk[4 * k + 3])
                     : "memory");
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full);
    }
    // epilogue: O / l -> fp16 row
    if (ok && sc.nT > 0) ok = waitb(&o_done, (sc.nT - 1) & 1, a.err, &abort_flag);
    if (__all_sync(0xffffffffu, ok) && sc.nT > 0) {
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.0f / l_run : 0.f;
      uint16_t* dst = a.out + (static_cast<size_t>(bq) * a.L + i) * D;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t u[32];
        tmem_ld32(trow + TM_O + 32 * c4, u);
        tmem_wait_ld();
        if (i < a.L) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w;
            w.x = pack_f16x2(__uint_as_float(u[e]) * inv, __uint_as_float(u[e + 1]) * inv);
            w.y = pack_f16x2(__uint_as_float(u[e + 2]) * inv, __uint_as_float(u[e + 3]) * inv);
            w.z = pack_f16x2(__uint_as_float(u[e + 4]) * inv, __uint_as_float(u[e + 5]) * inv);
            w.w = pack_f16x2(__uint_as_float(u[e + 6]) * inv, __uint_as_float(u[e + 7]) * inv);
            *reinterpret_cast<uint4*>(dst + 32 * c4 + e) = w;
          }
        }
      }
    }
  }
  __syncwarp();  // producer / MMA warps: lanes wait for their issuing lanes before the CTA barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ pre-pass

// One CTA (256 threads) per (128-position block, head, batch) of x [B, H, L, D]:
// scale = amax / 448 (1 when amax is 0); mode 0 writes e4m3 codes [B*H][Lp][D],
// mode 1 writes fp16(e4m3 value * scale); rows past L are zero.
__global__ void __launch_bounds__(256) fp8_block_quant(const uint16_t* __restrict__ x, int H, int L, int Lp, int nblk,
                                                       uint8_t* __restrict__ codes, uint16_t* __restrict__ vals,
                                                       float* __restrict__ scales) {
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * H + h;
  const int r0 = blk * 128;
  __shared__ float red[8];
  __shared__ float s_scale;
  // each thread: 4 rows x 16 columns as 8-byte loads of 4 halves
  float amax = 0.f;
  for (int e = threadIdx.x; e < 128 * 32; e += 256) {
    const int r = e >> 5, c4 = e & 31;
    const int row = r0 + r;
    if (row < L) {
      const uint2 u = reinterpret_cast<const uint2*>(x + (bh * L + row) * D)[c4];
      amax = fmaxf(amax, fabsf(__half2float(__ushort_as_half(static_cast<unsigned short>(u.x & 0xFFFFu)))));
      amax = fmaxf(amax, fabsf(__half2float(__ushort_as_half(static_cast<unsigned short>(u.x >> 16)))));
      amax = fmaxf(amax, fabsf(__half2float(__ushort_as_half(static_cast<unsigned short>(u.y & 0xFFFFu)))));
      amax = fmaxf(amax, fabsf(__half2float(__ushort_as_half(static_cast<unsigned short>(u.y >> 16)))));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w]);
    const float s = m == 0.f ? 1.0f : __fdiv_rn(m, E4M3_MAX);
    s_scale = s;
    scales[bh * nblk + blk] = s;
  }
  __syncthreads();
  const float s = s_scale;
  for (int e = threadIdx.x; e < 128 * 32; e += 256) {
    const int r = e >> 5, c4 = e & 31;
    const int row = r0 + r;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (row < L) {
      const uint2 u = reinterpret_cast<const uint2*>(x + (bh * L + row) * D)[c4];
      v[0] = __half2float(__ushort_as_half(static_cast<unsigned short>(u.x & 0xFFFFu)));
      v[1] = __half2float(__ushort_as_half(static_cast<unsigned short>(u.x >> 16)));
      v[2] = __half2float(__ushort_as_half(static_cast<unsigned short>(u.y & 0xFFFFu)));
      v[3] = __half2float(__ushort_as_half(static_cast<unsigned short>(u.y >> 16)));
    }
    uint32_t q[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) q[k] = __nv_cvt_float_to_fp8(__fdiv_rn(v[k], s), __NV_SATFINITE, __NV_E4M3);
    const size_t o = (bh * Lp + row) * D + 4 * c4;
    if (codes) {
      *reinterpret_cast<uint32_t*>(codes + o) = q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24);
    } else {
      uint32_t h2[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float a0 = __half2float(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(q[2 * k]), __NV_E4M3)) * s;
        const float a1 = __half2float(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(q[2 * k + 1]), __NV_E4M3)) * s;
        h2[k] = pack_f16x2(a0, a1);
      }
      *reinterpret_cast<uint2*>(vals + o) = make_uint2(h2[0], h2[1]);
    }
  }
}

// Score bias of the e4m3 key blocks, [B*Hkv][Lp]: 0 for positions < L, -inf past L
// (vl_prep then marks the vertical lines -inf too: they are read as fp16 tiles).
__global__ void kbias_init(float* __restrict__ kbias, int L, int Lp, size_t n) {
  for (size_t e = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<size_t>(gridDim.x) * blockDim.x)
    kbias[e] = static_cast<int>(e % Lp) < L ? 0.f : -INFINITY;
}

// Gathered VL rows of K and V and the -inf bias of their positions; grid
// (nvlp / 128, B*Hkv).  Row r of (b, kv head) holds position vl_pos[r] (r < n_vl)
// or zeros with position INT_MAX.
__global__ void vl_prep(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v, const int32_t* __restrict__ vl_pos,
                        int n_vl, int vl_stride, int L, int Lp, int nvlp, float* __restrict__ kbias,
                        uint16_t* __restrict__ kvl, uint16_t* __restrict__ vvl, int32_t* __restrict__ vlpos_pad) {
  const int bh = blockIdx.y;
  const int r0 = blockIdx.x * TKEY;
  for (int e = threadIdx.x; e < TKEY * (D / 8); e += blockDim.x) {
    const int r = r0 + e / (D / 8), ch = e % (D / 8);
    uint4 kk = make_uint4(0u, 0u, 0u, 0u), vv = make_uint4(0u, 0u, 0u, 0u);
    int pos = INT_MAX;
    if (r < n_vl) {
      const int p = vl_pos[static_cast<size_t>(bh) * vl_stride + r];
      if (p >= 0 && p < L) {
        pos = p;
        kk = reinterpret_cast<const uint4*>(k + (static_cast<size_t>(bh) * L + p) * D)[ch];
        vv = reinterpret_cast<const uint4*>(v + (static_cast<size_t>(bh) * L + p) * D)[ch];
        if (ch == 0) kbias[static_cast<size_t>(bh) * Lp + p] = -INFINITY;
      }
    }
    reinterpret_cast<uint4*>(kvl + (static_cast<size_t>(bh) * nvlp + r) * D)[ch] = kk;
    reinterpret_cast<uint4*>(vvl + (static_cast<size_t>(bh) * nvlp + r) * D)[ch] = vv;
    if (ch == 0) vlpos_pad[static_cast<size_t>(bh) * nvlp + r] = pos;
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D map over [z][y][x] rows of 128 elements; box {box_x, 128, 1}, 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, bool fp16, int rows, int heads, int box_x) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const int esz = fp16 ? 2 : 1;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(128 * esz), static_cast<cuuint64_t>(rows) * 128 * esz};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_x), 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct PfLayout {
  size_t err, q8, k8, v8, sq, sk, sv, kbias, kvl, vvl, vlpos, total;
  int Lp, nblk, nvlp;
};

PfLayout pf_layout(int B, int Hq, int Hkv, int L, int n_vl) {
  PfLayout l;
  l.Lp = ((L + 127) / 128) * 128;
  l.nblk = l.Lp / 128;
  l.nvlp = ((max(n_vl, 1) + 127) / 128) * 128;
  auto al = [](size_t x) { return (x + 1023) & ~static_cast<size_t>(1023); };
  size_t o = 0;
  l.err = o; o = al(o + 16);
  l.q8 = o; o = al(o + static_cast<size_t>(B) * Hq * l.Lp * D);
  l.k8 = o; o = al(o + static_cast<size_t>(B) * Hkv * l.Lp * D);
  l.v8 = o; o = al(o + static_cast<size_t>(B) * Hkv * l.Lp * D * 2);
  l.sq = o; o = al(o + static_cast<size_t>(B) * Hq * l.nblk * 4);
  l.sk = o; o = al(o + static_cast<size_t>(B) * Hkv * l.nblk * 4);
  l.sv = o; o = al(o + static_cast<size_t>(B) * Hkv * l.nblk * 4);
  l.kbias = o; o = al(o + static_cast<size_t>(B) * Hkv * l.Lp * 4);
  l.kvl = o; o = al(o + static_cast<size_t>(B) * Hkv * l.nvlp * D * 2);
  l.vvl = o; o = al(o + static_cast<size_t>(B) * Hkv * l.nvlp * D * 2);
  l.vlpos = o; o = al(o + static_cast<size_t>(B) * Hkv * l.nvlp * 4);
  l.total = o;
  return l;
}

}  // namespace

// Workspace for any VL set of up to L positions.  Bytes [0, 4) of the workspace
// receive the kernel's error word (non-zero if a bounded wait gave up).
size_t prefill_workspace(int B, int Hq, int Hkv, int L) { return pf_layout(B, Hq, Hkv, L, L).total; }

hq_status launch_prefill(int B, int Hq, int Hkv, int L, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const int32_t* vl_pos, int n_vl, int vl_stride, int W, float sm_scale, uint16_t* out, void* ws,
                         cudaStream_t st) {
  if (n_vl > L) return HQ_ERR_INVALID;
  const PfLayout ly = pf_layout(B, Hq, Hkv, L, n_vl);
  char* w = static_cast<char*>(ws);
  uint32_t* err = reinterpret_cast<uint32_t*>(w + ly.err);
  uint8_t* q8 = reinterpret_cast<uint8_t*>(w + ly.q8);
  uint8_t* k8 = reinterpret_cast<uint8_t*>(w + ly.k8);
  uint16_t* v8 = reinterpret_cast<uint16_t*>(w + ly.v8);
  float* sq = reinterpret_cast<float*>(w + ly.sq);
  float* sk = reinterpret_cast<float*>(w + ly.sk);
  float* sv = reinterpret_cast<float*>(w + ly.sv);
  float* kbias = reinterpret_cast<float*>(w + ly.kbias);
  uint16_t* kvl = reinterpret_cast<uint16_t*>(w + ly.kvl);
  uint16_t* vvl = reinterpret_cast<uint16_t*>(w + ly.vvl);
  int32_t* vlpos = reinterpret_cast<int32_t*>(w + ly.vlpos);

  Tmaps tm;
  if (!make_map(&tm.q8, q8, false, ly.Lp, B * Hq, 128) || !make_map(&tm.q16, q, true, L, B * Hq, 64) ||
      !make_map(&tm.k8, k8, false, ly.Lp, B * Hkv, 128) || !make_map(&tm.v8, v8, true, ly.Lp, B * Hkv, 64) ||
      !make_map(&tm.k16, k, true, L, B * Hkv, 64) || !make_map(&tm.v16, v, true, L, B * Hkv, 64) ||
      !make_map(&tm.kvl, kvl, true, ly.nvlp, B * Hkv, 64) || !make_map(&tm.vvl, vvl, true, ly.nvlp, B * Hkv, 64))
    return cuda_fail(cudaSuccess, "prefill tensor maps");

  if (cudaMemsetAsync(err, 0, 16, st) != cudaSuccess) return cuda_fail(cudaGetLastError(), "prefill setup");
  kbias_init<<<256, 256, 0, st>>>(kbias, L, ly.Lp, static_cast<size_t>(B) * Hkv * ly.Lp);
  fp8_block_quant<<<dim3(ly.nblk, Hq, B), 256, 0, st>>>(q, Hq, L, ly.Lp, ly.nblk, q8, nullptr, sq);
  fp8_block_quant<<<dim3(ly.nblk, Hkv, B), 256, 0, st>>>(k, Hkv, L, ly.Lp, ly.nblk, k8, nullptr, sk);
  fp8_block_quant<<<dim3(ly.nblk, Hkv, B), 256, 0, st>>>(v, Hkv, L, ly.Lp, ly.nblk, nullptr, v8, sv);
  vl_prep<<<dim3(ly.nvlp / TKEY, B * Hkv), 256, 0, st>>>(k, v, vl_pos, n_vl, vl_stride, L, ly.Lp, ly.nvlp, kbias, kvl, vvl,
                                                         vlpos);
  PfArgs a;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.L = L; a.Lp = ly.Lp; a.nblk = ly.nblk; a.W = W; a.n_vl = n_vl; a.nvlp = ly.nvlp;
  a.qk_scale = sm_scale * LOG2E;
  a.sq = sq; a.sk = sk; a.kbias = kbias; a.vlpos = vlpos; a.out = out; a.err = err;
  int dev = 0;
  cudaGetDevice(&dev);
  static bool attr_done[64] = {};
  if (dev >= 64 || !attr_done[dev]) {
    if (cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PF_SMEM) != cudaSuccess)
      return cuda_fail(cudaGetLastError(), "prefill setup");
    if (dev < 64) attr_done[dev] = true;
  }
  prefill_kernel<<<dim3(ly.nblk, Hq, B), PF_THREADS, PF_SMEM, st>>>(tm, a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    // name the kernel's resources in the message (launch-resource failures)
    cudaFuncAttributes fa;
    char where[120] = "prefill launch";
    if (cudaFuncGetAttributes(&fa, prefill_kernel) == cudaSuccess)
      snprintf(where, sizeof(where), "prefill launch (regs %d, local %zu B, static smem %zu B, max threads %d)", fa.numRegs,
               fa.localSizeBytes, fa.sharedSizeBytes, fa.maxThreadsPerBlock);
    return cuda_fail(e, where);
  }
  return HQ_OK;
}

}  // namespace hq
