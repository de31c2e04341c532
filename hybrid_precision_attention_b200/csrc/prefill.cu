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
//                                              (b, head, 128 positions): x8 = e4m3(x / s);
//                                              or (INT8-QK format) INT8 Q, K, scale amax / 127,
//                                              and FP16 V
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
//   prefill_kernel   one CTA per (pair of 128-query tiles, query head, batch),
//                    longest rows first; both query tiles share every K / V tile:
//                      warps 0-7  two softmax warpgroups, one per query tile, one
//                                 query row per thread = one TMEM lane
//                      warp 8     TMA producers: lane 0 both query tiles once and
//                                 the K tiles (with their score bias or VL
//                                 positions and K scales), lane 1 the V tiles
//                      warp 9     TMEM allocation and the tcgen05.mma issue,
//                                 event-driven over the four MMAs of a tile
//                    key tiles in order: VL tiles and the window's tiles first
//                    (QK on kind::f16 with the fp16 queries), then the e4m3 tiles
//                    (QK on kind::f8f6f4); once the fp16 tiles are done, the
//                    64 KB of fp16 queries serve as a second K / V stage.  S = Q K^T
//                    of each query tile lands in its own TMEM columns; its softmax
//                    group reads S, writes P (fp16) to shared memory in the
//                    128-byte-swizzled K-major layout, and O += P V (kind::f16,
//                    V MN-major) accumulates in TMEM.  One pass per tile against
//                    the running max; only when a row sum leaves 2^8 (every row's
//                    first tile, rarely later) is the exact tile max taken, O
//                    rescaled and P recomputed.
// All mbarrier waits are bounded (about 1 s); a timeout sets the error word and
// the CTA drains its copies and MMAs before releasing TMEM.
#include <climits>
#include <cstdio>
#include <cuda_fp8.h>

#include "tc.cuh"

namespace hq {
namespace {

constexpr int TQ = 128, TKEY = 128;
constexpr int PF_THREADS = 320;                 // 2 softmax warpgroups, a TMA warp, an MMA warp
constexpr int W_TMA = 8, W_MMA = 9;
constexpr float E4M3_MAX = 448.0f;
// shared memory map (byte offsets from a 1024-byte aligned base); the CTA holds
// two query tiles (A: rows q0 .. q0+127, B: q0+128 .. q0+255) that share every
// K / V tile.  The fp16 query tiles are needed only by the fp16 key tiles, which
// come first; afterwards their 64 KB hold a second K / V stage.
constexpr int SM_Q8 = 0;                        // Q e4m3  2 tiles x [128][128 B]             32 KB
constexpr int SM_Q16 = 32768;                   // Q fp16  2 tiles x 2 x [128][128 B]         64 KB  (later K / V stage 1)
constexpr int SM_K = SM_Q16 + 65536;            // K stage 0 (e4m3 tiles use the first 16 KB)  32 KB
constexpr int SM_V = SM_K + 32768;              // V stage 0 fp16 2 x [128 keys][128 B]        32 KB
constexpr int SM_P = SM_V + 32768;              // P fp16  2 tiles x 2 x [128][128 B]          64 KB
constexpr int SM_AUX = SM_P + 65536;            // 2 stages x 512 B: mask bias (e4m3 tiles) or VL positions
constexpr int SM_KS = SM_AUX + 1024;            // 2 stages x 16 B: the 16-byte chunk holding the e4m3 tile's K scale
constexpr int SM_USED = SM_KS + 32;
constexpr int PF_SMEM = SM_USED + 1024;         // + slack for the 1024-byte alignment
constexpr uint32_t TMEM_COLS = 512;             // S_A 0..127, S_B 128..255, O_A 256..383, O_B 384..511
constexpr uint32_t TM_S = 0, TM_O = 256;
constexpr uint32_t IDESC_QK = idesc_make(0, 0, 0, TQ, TKEY);   // K-major A and B
constexpr uint32_t IDESC_QK_I8 = idesc_i8_make(TQ, TKEY);      // INT8 Q.K, s32 accumulate
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
  int int_qk;            // quantised tiles: INT8 Q.K (s32 in TMEM) and FP16 V, else e4m3 Q, K, V
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

// per-CTA tile schedule (the union of what the two query tiles need)
struct Sched {
  int pr, q0, imax, nA, nB, nC, ktw0, nvv, nT;
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
  s.pr = gridDim.x - 1 - blockIdx.x;  // longest rows first
  s.q0 = s.pr * 2 * TQ;
  s.imax = min(s.q0 + 2 * TQ - 1, a.L - 1);
  const int jmax = s.imax - a.W;  // largest key any row of the pair sees outside its window
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

// Tile order of a CTA: [0, nB) VL tiles, [nB, nF) the window's fp16 key blocks
// from ktw0 (nF = nB + nC), then [nF, nT) the e4m3 key blocks 0 .. nA-1.
// Stages: the fp16 tiles all use stage 0; e4m3 tile nF + j uses stage j % 2
// (stage 1 lives where the fp16 query tiles were).  use = how many tiles used
// the stage before this one (its barrier phase).
struct TileSlot {
  int stage, use, prev;  // prev: the tile that used the stage before (-1: none)
};
__device__ __forceinline__ TileSlot slot_of(int t, int nF) {
  TileSlot z;
  if (t < nF) {
    z.stage = 0;
    z.use = t;
    z.prev = t - 1;
  } else {
    const int j = t - nF;
    z.stage = j & 1;
    z.use = z.stage == 0 ? nF + j / 2 : j / 2;
    z.prev = j >= 2 ? t - 2 : (z.stage == 0 ? nF - 1 : -1);
  }
  return z;
}

// Scale and mask 32 scores of row i (columns c0 .. c0+31 of tile t) in place;
// returns their max.  Columns a row must not see become -inf.
template <bool MAX>
__device__ __forceinline__ float scale_mask32(float (&x)[32], int c0, int t, const Sched& sc, const PfArgs& a,
                                              const uint8_t* aux, float scl, int i) {
  float mt = -INFINITY;
  const int nF = sc.nB + sc.nC;
  if (t >= nF) {
    float bv[32];
#pragma unroll
    for (int c4 = 0; c4 < 8; ++c4) {
      const float4 bb = reinterpret_cast<const float4*>(aux)[c0 / 4 + c4];
      bv[4 * c4] = bb.x;
      bv[4 * c4 + 1] = bb.y;
      bv[4 * c4 + 2] = bb.z;
      bv[4 * c4 + 3] = bb.w;
    }
    const int jlim = i - a.W - (t - nF) * TKEY - c0;  // causal limit: local columns c <= jlim
    if (a.int_qk) {
      // s32 accumulators: exact to float by the 1.5 * 2^23 bias (|Q.K| < 128 * 127 * 127 < 2^22)
#pragma unroll
      for (int c = 0; c < 32; ++c) x[c] = __uint_as_float(__float_as_uint(x[c]) + 0x4B400000u) - 12582912.0f;
    }
    float m2[2] = {-INFINITY, -INFINITY};
    if (jlim >= 31) {
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        x[c] = fmaf(x[c], scl, bv[c]);
        if (MAX) m2[c & 1] = fmaxf(m2[c & 1], x[c]);
      }
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        x[c] = c <= jlim ? fmaf(x[c], scl, bv[c]) : -INFINITY;
        if (MAX) m2[c & 1] = fmaxf(m2[c & 1], x[c]);
      }
    }
    if (MAX) mt = fmaxf(m2[0], m2[1]);
  } else if (t < sc.nB) {
    const int32_t* vp = reinterpret_cast<const int32_t*>(aux) + c0;
    const int lim = i - a.W;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      x[c] = vp[c] <= lim ? x[c] * a.qk_scale : -INFINITY;
      if (MAX) mt = fmaxf(mt, x[c]);
    }
  } else {
    const int kt = sc.ktw0 + (t - sc.nB);
    const int lo = i - a.W + 1 - kt * TKEY - c0, hi = i - kt * TKEY - c0;  // window: lo <= c <= hi
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      x[c] = (c >= lo && c <= hi) ? x[c] * a.qk_scale : -INFINITY;
      if (MAX) mt = fmaxf(mt, x[c]);
    }
  }
  return mt;
}

// Per tile (all waits bounded):
//   K lane   K(t) + aux into its stage once QK_A, QK_B of the stage's previous
//            tile are done and both softmax groups have read that tile's aux
//   V lane   V(t) into its stage once PV_A, PV_B of the stage's previous tile are done
//   MMA      event-driven: QK_g(t) when K(t) landed and group g has read S_g(t-1);
//            PV_g(t) when P_g(t) and V(t) landed
//   softmax  group g, one pass over S_g(t): scale, mask, exp2 against the
//            running max, P_g(t) to shared memory; only when a row's tile max
//            exceeds its running max by more than 2^8 (every row's first
//            tile, rarely later) is the pass redone with the new max and O_g
//            rescaled
__global__ void __launch_bounds__(PF_THREADS, 1) prefill_kernel(const __grid_constant__ Tmaps tm, const PfArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t q_full, q16_free, drain, k_full[2], k_empty[2], aux_free[2], v_full[2], v_empty[2],
      s_full[2], s_free[2], p_full[2], o_done[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int hq = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  const int kvh = hq / G;
  const int bq = b * a.Hq + hq, bk = b * a.Hkv + kvh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Sched sc = schedule(a, bk);
  const int nF = sc.nB + sc.nC;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&q16_free, 1);
    mbar_init(&drain, 1);
    for (int g = 0; g < 2; ++g) {
      mbar_init(&k_full[g], 1);
      mbar_init(&k_empty[g], 1);
      mbar_init(&aux_free[g], 256);
      mbar_init(&v_full[g], 1);
      mbar_init(&v_empty[g], 1);
      mbar_init(&s_full[g], 1);
      mbar_init(&s_free[g], 128);
      mbar_init(&p_full[g], 128);
      mbar_init(&o_done[g], 1);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == W_MMA) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t sm_base = smem_u32(sm);
  auto k_stage = [&](int st) -> uint32_t { return st == 0 ? SM_K : SM_Q16; };
  auto v_stage = [&](int st) -> uint32_t { return st == 0 ? SM_V : SM_Q16 + 32768; };

  if (warp == W_TMA) {
    // ------------------------------------------------------------ TMA producers
    // lane 0: both query tiles once, then the K tiles with their auxiliary data;
    // lane 1: the V tiles.  The two lanes wait on different barriers.
    if (lane == 0) {
      mbar_arrive_expect_tx(&q_full, 2 * (16384 + 32768));
      for (int g = 0; g < 2; ++g) {
        const int qr = sc.q0 + g * TQ;
        tma_load_3d(sm + SM_Q8 + g * 16384, &tm.q8, 0, qr, bq, &q_full);
        tma_load_3d(sm + SM_Q16 + g * 32768, &tm.q16, 0, qr, bq, &q_full);
        tma_load_3d(sm + SM_Q16 + g * 32768 + 16384, &tm.q16, 64, qr, bq, &q_full);
      }
      int issued[2] = {0, 0};
      bool ok = true;
      for (int t = 0; ok && t < sc.nT; ++t) {
        const TileSlot z = slot_of(t, nF);
        // the stage is free once both QKs of its previous tile are done and both
        // softmax groups have read that tile's aux (barriers counted per use of
        // the stage, so a wait is never more than one phase behind)
        if (z.prev >= 0) {
          const int pu = slot_of(z.prev, nF).use;
          ok = waitb(&k_empty[z.stage], pu & 1, a.err, &abort_flag) && waitb(&aux_free[z.stage], pu & 1, a.err, &abort_flag);
        }
        if (ok && t == nF) {
          // every fp16 QK is done (the stage-0 wait above) and the fp16 query
          // tiles have landed: their region may now serve as stage 1
          ok = waitb(&q_full, 0, a.err, &abort_flag);
          if (ok) mbar_arrive(&q16_free);
        }
        if (!ok) break;
        uint8_t* K = sm + k_stage(z.stage);
        uint8_t* aux = sm + SM_AUX + z.stage * 512;
        if (t >= nF) {
          const int kt = t - nF;
          mbar_arrive_expect_tx(&k_full[z.stage], 16384 + 512 + 16);
          tma_load_3d(K, &tm.k8, 0, kt * TKEY, bk, &k_full[z.stage]);
          bulk_g2s(aux, a.kbias + static_cast<size_t>(bk) * a.Lp + kt * TKEY, 512, &k_full[z.stage]);
          bulk_g2s(sm + SM_KS + z.stage * 16, a.sk + ((static_cast<size_t>(bk) * a.nblk + kt) & ~static_cast<size_t>(3)), 16,
                   &k_full[z.stage]);
        } else if (t < sc.nB) {
          mbar_arrive_expect_tx(&k_full[0], 32768 + 512);
          tma_load_3d(K, &tm.kvl, 0, t * TKEY, bk, &k_full[0]);
          tma_load_3d(K + 16384, &tm.kvl, 64, t * TKEY, bk, &k_full[0]);
          bulk_g2s(aux, a.vlpos + static_cast<size_t>(bk) * a.nvlp + t * TKEY, 512, &k_full[0]);
        } else {
          const int kt = sc.ktw0 + (t - sc.nB);
          mbar_arrive_expect_tx(&k_full[0], 32768);
          tma_load_3d(K, &tm.k16, 0, kt * TKEY, bk, &k_full[0]);
          tma_load_3d(K + 16384, &tm.k16, 64, kt * TKEY, bk, &k_full[0]);
        }
        issued[z.stage] = z.use + 1;
      }
      if (abort_flag) {
        // never expected: let every issued copy land before the CTA can exit
        int dummy = 0;
        for (int st = 0; st < 2; ++st)
          if (issued[st] > 0) waitb(&k_full[st], (issued[st] - 1) & 1, a.err, &dummy);
        waitb(&q_full, 0, a.err, &dummy);
      }
    } else if (lane == 1) {
      int issued[2] = {0, 0};
      bool ok = true;
      for (int t = 0; ok && t < sc.nT; ++t) {
        const TileSlot z = slot_of(t, nF);
        if (z.prev >= 0) ok = waitb(&v_empty[z.stage], slot_of(z.prev, nF).use & 1, a.err, &abort_flag);
        // V stage 1 is the second fp16 query tile: free once the K lane says so
        if (ok && z.stage == 1 && z.use == 0) ok = waitb(&q16_free, 0, a.err, &abort_flag);
        if (!ok) break;
        uint8_t* V = sm + v_stage(z.stage);
        const CUtensorMap* map;
        int row;
        if (t >= nF) {
          map = &tm.v8;
          row = (t - nF) * TKEY;
        } else if (t < sc.nB) {
          map = &tm.vvl;
          row = t * TKEY;
        } else {
          map = &tm.v16;
          row = (sc.ktw0 + (t - sc.nB)) * TKEY;
        }
        mbar_arrive_expect_tx(&v_full[z.stage], 32768);
        tma_load_3d(V, map, 0, row, bk, &v_full[z.stage]);
        tma_load_3d(V + 16384, map, 64, row, bk, &v_full[z.stage]);
        issued[z.stage] = z.use + 1;
      }
      if (abort_flag) {
        int dummy = 0;
        for (int st = 0; st < 2; ++st)
          if (issued[st] > 0) waitb(&v_full[st], (issued[st] - 1) & 1, a.err, &dummy);
      }
    }
  } else if (warp == W_MMA) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      bool ok = waitb(&q_full, 0, a.err, &abort_flag);
      auto issue_qk = [&](int g, int t, int st) {
        tc_fence_after();
        const uint32_t S = tmem + TM_S + 128 * g;
        const uint32_t K = sm_base + k_stage(st);
        if (t >= nF) {
          const uint32_t q8 = sm_base + SM_Q8 + g * 16384;
          if (a.int_qk) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_i8(S, sdesc_sw128(q8 + 32 * kk, 16, 1024), sdesc_sw128(K + 32 * kk, 16, 1024), IDESC_QK_I8, kk > 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f8(S, sdesc_sw128(q8 + 32 * kk, 16, 1024), sdesc_sw128(K + 32 * kk, 16, 1024), IDESC_QK, kk > 0);
          }
        } else {
          const uint32_t q16 = sm_base + SM_Q16 + g * 32768;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + 32 * (kk & 3);
            umma_f16(S, sdesc_sw128(q16 + off, 16, 1024), sdesc_sw128(K + off, 16, 1024), IDESC_QK, kk > 0);
          }
        }
        umma_commit(&s_full[g]);
      };
      auto issue_pv = [&](int g, int t, int st) {
        tc_fence_after();
        const uint32_t p = sm_base + SM_P + g * 32768;
        const uint32_t V = sm_base + v_stage(st);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * 16384 + 32 * (kk & 3);
          umma_f16(tmem + TM_O + 128 * g, sdesc_sw128(p + aoff, 16, 1024), sdesc_sw128(V + 2048 * kk, 16384, 1024),
                   IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&o_done[g]);
      };
      // Event-driven issue: whichever of QK_A, QK_B, PV_A, PV_B is ready goes
      // next.  The groups stay within a stage's reuse distance of each other,
      // which keeps every probed barrier within one phase.
      int tq[2] = {0, 0}, tp[2] = {0, 0};
      uint64_t t_last = global_ns();
      while (ok && (tp[0] < sc.nT || tp[1] < sc.nT)) {
        bool progress = false;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const int t = tq[g];
          if (t < sc.nT) {
            const TileSlot z = slot_of(t, nF);
            if (mbar_test_wait(&k_full[z.stage], z.use & 1) && (t == 0 || mbar_test_wait(&s_free[g], (t - 1) & 1))) {
              issue_qk(g, t, z.stage);
              if (tq[g ^ 1] > t) umma_commit(&k_empty[z.stage]);  // both QKs of tile t issued
              tq[g] = t + 1;
              progress = true;
            }
          }
          const int u = tp[g];
          if (u < tq[g]) {
            const TileSlot z = slot_of(u, nF);
            if (mbar_test_wait(&p_full[g], u & 1) && mbar_test_wait(&v_full[z.stage], z.use & 1)) {
              issue_pv(g, u, z.stage);
              if (tp[g ^ 1] > u) umma_commit(&v_empty[z.stage]);  // both PVs of tile u issued
              tp[g] = u + 1;
              progress = true;
            }
          }
        }
        if (progress) {
          t_last = global_ns();
        } else if (*reinterpret_cast<volatile int*>(&abort_flag)) {
          ok = false;
        } else if (global_ns() - t_last > 1000000000ull) {
          atomicOr(a.err, 1u);
          abort_flag = 1;
          ok = false;
        }
      }
      // every MMA this thread issued completes before TMEM is released
      umma_commit(&drain);
      int dummy = 0;
      waitb(&drain, 0, a.err, &dummy);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0..7)
    const int g = warp >> 2;          // query tile of this warpgroup
    const int r = threadIdx.x & 127;  // row within the tile = TMEM lane
    const int i = sc.q0 + g * TQ + r;
    const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t srow = trow + TM_S + 128 * g, orow = trow + TM_O + 128 * g;
    const uint32_t prow = sm_base + SM_P + g * 32768 + r * 128;
    float m_run = -INFINITY, l_run = 0.f;
    // tile B of the last pair may lie wholly past L (its rows are never stored)
    const float sqv = a.sq[static_cast<size_t>(bq) * a.nblk + min(sc.pr * 2 + g, a.nblk - 1)];
    bool ok = true;
    for (int t = 0; t < sc.nT; ++t) {
      const TileSlot z = slot_of(t, nF);
      const uint8_t* aux = sm + SM_AUX + z.stage * 512;
      ok = ok && waitb(&s_full[g], t & 1, a.err, &abort_flag);
      // P_g is read by PV_g(t-1): wait for it before storing this tile's P
      if (t > 0) ok = ok && waitb(&o_done[g], (t - 1) & 1, a.err, &abort_flag);
      if (!__all_sync(0xffffffffu, ok)) ok = false;
      if (!ok) break;
      tc_fence_after();
      const float scl = t >= nF ? sqv * reinterpret_cast<const float*>(sm + SM_KS + z.stage * 16)
                                           [(static_cast<size_t>(bk) * a.nblk + (t - nF)) & 3] * a.qk_scale
                                : a.qk_scale;
      // One pass per tile: P = exp2(s - m_run) against the running max, the
      // row sum in fp32.  A row sum above 2^8 (or not finite) means some p may
      // have left the safe fp16 range because the row's max moved up: only then
      // is the tile's exact max taken (another pass over S), the running max
      // moved, O rescaled and P recomputed (p <= 2^8 otherwise, and the sum and
      // O accumulate in fp32).
      float lt = 0.f;
      // a row without a running max yet (its first tile, or all keys so far
      // masked) takes the exact-max path directly
      const int pass_first = __any_sync(0xffffffffu, m_run == -INFINITY) ? 1 : 0;
      for (int pass = pass_first; pass < 3; ++pass) {
        if (pass == 1) {
          // the exact row max of this tile
          float mt = -INFINITY;
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            float x[32];
            tmem_ld32f(srow + 32 * c4, x);
            tmem_wait_ld();
            mt = fmaxf(mt, scale_mask32<true>(x, 32 * c4, t, sc, a, aux, scl, i));
          }
          const bool grow = mt > m_run;
          float alpha = 1.f;
          if (grow) {
            alpha = m_run != -INFINITY ? ex2(m_run - mt) : 0.f;
            m_run = mt;
            l_run *= alpha;
          }
          // the TMEM accesses are warp-collective (.sync.aligned): the whole warp
          // rescales its O rows, rows whose max did not move by 1
          if (t > 0) {
#pragma unroll 1
            for (int c4 = 0; c4 < 4; ++c4) {
              uint32_t u[32];
              tmem_ld32(orow + 32 * c4, u);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
              tmem_st32(orow + 32 * c4, u);
            }
            tmem_wait_st();
          }
          continue;
        }
        // P = exp2(s - m_run) in fp16 into shared memory (K-major, 128-byte
        // swizzle: 16-byte chunk k of the row goes to chunk k ^ (r % 8) of its
        // 128-byte line; keys 64..127 in region 1), row sum in fp32
        const float mref = m_run == -INFINITY ? 0.f : m_run;
        float l0 = 0.f, l1 = 0.f;
        float x[32];
        tmem_ld32f(srow, x);
        tmem_wait_ld();
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          scale_mask32<false>(x, 32 * c4, t, sc, a, aux, scl, i);
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float p0 = ex2(x[c] - mref), p1 = ex2(x[c + 1] - mref);
            l0 += p0;
            l1 += p1;
            pk[c / 2] = pack_f16x2(p0, p1);
          }
          if (c4 < 3) tmem_ld32f(srow + 32 * (c4 + 1), x);  // next chunk in flight during the stores
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int kc = 4 * c4 + k;  // 16-byte chunk of the row (8 keys)
            const uint32_t addr = prow + (kc >> 3) * 16384 + ((((kc & 7) ^ (r & 7))) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * k]), "r"(pk[4 * k + 1]),
                         "r"(pk[4 * k + 2]), "r"(pk[4 * k + 3])
                         : "memory");
          }
          if (c4 < 3) tmem_wait_ld();
        }
        lt = l0 + l1;
        if (pass == 2) break;
        const bool grow = !(lt <= 256.0f);  // also true for inf / NaN
        if (!__any_sync(0xffffffffu, grow)) break;
      }
      l_run += lt;
      // S_g(t) and the stage's auxiliary data have been read for the last time
      tc_fence_before();
      mbar_arrive(&s_free[g]);
      mbar_arrive(&aux_free[z.stage]);
      fence_proxy_async_smem();
      mbar_arrive(&p_full[g]);
    }
    // epilogue: O / l -> fp16 row
    if (ok && sc.nT > 0) ok = waitb(&o_done[g], (sc.nT - 1) & 1, a.err, &abort_flag);
    if (__all_sync(0xffffffffu, ok) && sc.nT > 0) {
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.0f / l_run : 0.f;
      uint16_t* dst = a.out + (static_cast<size_t>(bq) * a.L + i) * D;
#pragma unroll 1
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t u[32];
        tmem_ld32(orow + 32 * c4, u);
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
  if (warp == W_MMA) {
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

// INT8 pre-pass (INT8-QK format): one CTA (256 threads) per (128-position
// block, head, batch) of x [B, H, L, D]: scale = amax / 127 (1 when amax is 0),
// codes clamp(rint_even(x / scale), -127, 127) [B*H][Lp][D]; rows past L are zero.
__global__ void __launch_bounds__(256) int8_block_quant(const uint16_t* __restrict__ x, int H, int L, int Lp, int nblk,
                                                        int8_t* __restrict__ codes, float* __restrict__ scales) {
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * H + h;
  const int r0 = blk * 128;
  __shared__ float red[8];
  __shared__ float s_scale;
  float amax = 0.f;
  for (int e = threadIdx.x; e < 128 * 32; e += 256) {
    const int row = r0 + (e >> 5), c4 = e & 31;
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
    const float s = m == 0.f ? 1.0f : __fdiv_rn(m, 127.0f);
    s_scale = s;
    scales[bh * nblk + blk] = s;
  }
  __syncthreads();
  const float s = s_scale;
  for (int e = threadIdx.x; e < 128 * 32; e += 256) {
    const int row = r0 + (e >> 5), c4 = e & 31;
    uint32_t packed = 0u;
    if (row < L) {
      const uint2 u = reinterpret_cast<const uint2*>(x + (bh * L + row) * D)[c4];
      const float v[4] = {__half2float(__ushort_as_half(static_cast<unsigned short>(u.x & 0xFFFFu))),
                          __half2float(__ushort_as_half(static_cast<unsigned short>(u.x >> 16))),
                          __half2float(__ushort_as_half(static_cast<unsigned short>(u.y & 0xFFFFu))),
                          __half2float(__ushort_as_half(static_cast<unsigned short>(u.y >> 16)))};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int qv = min(max(__float2int_rn(__fdiv_rn(v[k], s)), -127), 127);
        packed |= (static_cast<uint32_t>(qv) & 0xFFu) << (8 * k);
      }
    }
    *reinterpret_cast<uint32_t*>(codes + (bh * Lp + row) * D + 4 * c4) = packed;
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

// Workspace for any VL set of up to vl_stride positions.  Bytes [0, 4) of the
// workspace receive the kernel's error word (non-zero if a bounded wait gave up).
size_t prefill_workspace(int B, int Hq, int Hkv, int L, int vl_stride) {
  return pf_layout(B, Hq, Hkv, L, min(max(vl_stride, 0), L)).total;
}

hq_status launch_prefill(int B, int Hq, int Hkv, int L, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const int32_t* vl_pos, int n_vl, int vl_stride, int W, int qk_format, float sm_scale,
                         uint16_t* out, void* ws, cudaStream_t st) {
  const bool int_qk = qk_format == HQ_PREFILL_INT8_QK;
  if (n_vl > L || n_vl > vl_stride) return HQ_ERR_INVALID;
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
      !make_map(&tm.k8, k8, false, ly.Lp, B * Hkv, 128) ||
      // quantised tiles' V: e4m3 values stored as fp16, or (INT8-QK) V itself
      !(int_qk ? make_map(&tm.v8, v, true, L, B * Hkv, 64) : make_map(&tm.v8, v8, true, ly.Lp, B * Hkv, 64)) ||
      !make_map(&tm.k16, k, true, L, B * Hkv, 64) || !make_map(&tm.v16, v, true, L, B * Hkv, 64) ||
      !make_map(&tm.kvl, kvl, true, ly.nvlp, B * Hkv, 64) || !make_map(&tm.vvl, vvl, true, ly.nvlp, B * Hkv, 64))
    return cuda_fail(cudaSuccess, "prefill tensor maps");

  if (cudaMemsetAsync(err, 0, 16, st) != cudaSuccess) return cuda_fail(cudaGetLastError(), "prefill setup");
  kbias_init<<<256, 256, 0, st>>>(kbias, L, ly.Lp, static_cast<size_t>(B) * Hkv * ly.Lp);
  if (int_qk) {
    int8_block_quant<<<dim3(ly.nblk, Hq, B), 256, 0, st>>>(q, Hq, L, ly.Lp, ly.nblk, reinterpret_cast<int8_t*>(q8), sq);
    int8_block_quant<<<dim3(ly.nblk, Hkv, B), 256, 0, st>>>(k, Hkv, L, ly.Lp, ly.nblk, reinterpret_cast<int8_t*>(k8), sk);
  } else {
    fp8_block_quant<<<dim3(ly.nblk, Hq, B), 256, 0, st>>>(q, Hq, L, ly.Lp, ly.nblk, q8, nullptr, sq);
    fp8_block_quant<<<dim3(ly.nblk, Hkv, B), 256, 0, st>>>(k, Hkv, L, ly.Lp, ly.nblk, k8, nullptr, sk);
    fp8_block_quant<<<dim3(ly.nblk, Hkv, B), 256, 0, st>>>(v, Hkv, L, ly.Lp, ly.nblk, nullptr, v8, sv);
  }
  vl_prep<<<dim3(ly.nvlp / TKEY, B * Hkv), 256, 0, st>>>(k, v, vl_pos, n_vl, vl_stride, L, ly.Lp, ly.nvlp, kbias, kvl, vvl,
                                                         vlpos);
  PfArgs a;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.L = L; a.Lp = ly.Lp; a.nblk = ly.nblk; a.W = W; a.n_vl = n_vl; a.nvlp = ly.nvlp;
  a.qk_scale = sm_scale * LOG2E;
  a.sq = sq; a.sk = sk; a.kbias = kbias; a.vlpos = vlpos; a.out = out; a.err = err;
  a.int_qk = int_qk ? 1 : 0;
  int dev = 0;
  cudaGetDevice(&dev);
  static DeviceOnce attrs;
  const cudaError_t ea = attrs.run(
      dev, [] { return cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PF_SMEM); });
  if (ea != cudaSuccess) return cuda_fail(ea, "prefill setup");
  prefill_kernel<<<dim3((ly.nblk + 1) / 2, Hq, B), PF_THREADS, PF_SMEM, st>>>(tm, a);
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
