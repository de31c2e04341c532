// decode.cu — one decode step of attention over the hybrid K4V4 / FP16 cache.
//
// HyQuant digest (agihunt.info), prefill/decode paragraph, and the repository
// README, Overview item 3: the decode cache stores most positions K4V4 and the
// vertical-line and recent positions FP16, and dequantisation is fused into the
// attention scan (online softmax over quantised blocks) so no FP16 cache is
// materialised.  The pages' kernel is Triton for SM80+; this is a B200 design.
//
// Design (bandwidth-bound: ~160 B of K4V4 per token and kv head):
//   * grid = (splits S, Hkv, B), one wave (a wide CTA per SM, or 3 narrow CTAs
//     per SM for large batches); every
//     CTA owns one GQA group (all G <= 8 query heads of a kv head share one
//     pass over the bytes) and a contiguous range of the head's tile list:
//     packed tiles (one page of 64 positions: 4 KB K codes, 4 KB V codes,
//     1 KB + 1 KB scale/zero, the VL bitmap), VL tiles (16 FP16 rows of the VL
//     store), ring tiles (16 slots of the FP16 ring, which is a multiple of 16
//     long, so a tile is one contiguous copy) and a last tile holding the new
//     token read straight from its input pointer;
//   * a producer warp streams tiles into a 2 NC-stage shared-memory ring with
//     large 1-D bulk async copies (cp.async.bulk, mbarrier completion, no
//     multicast): 1 copy per packed tile, 2 per FP16 tile;
//   * NC consumer warps take whole tiles round-robin, each owning 2 of the 2 NC
//     stages (tile i -> stage i % 2NC -> warp i % NC), so every stage has a
//     single consumer and a waiter is never a full barrier phase behind; every
//     split gets an even share of the packed tiles and an even share of the
//     FP16 tiles, so both its bytes and its arithmetic are balanced.  Nibbles
//     become fp16 in registers (exponent-bias trick + one fma with the group's
//     scale/zero), and
//     both products run on tensor cores with mma.m16n8k16 (f32 accumulate):
//       S^T[keys x 8 queries] = K^ (16 keys x 16 dims) . Q^T
//       O^T[dims x 8 queries] += V^T (16 dims x 16 keys) . P^T
//     P^T comes from the S^T accumulators by an 8x8 movmatrix transpose.  Dims
//     and keys are permuted inside each MMA so that every thread dequantises one
//     whole group from contiguous nibbles and the packed-tile shared-memory
//     reads are free of bank conflicts;
//   * per-warp online softmax in the exp2 domain, a CTA merge in shared memory,
//     then split partials (m, l, O) go to the workspace and the last CTA of each
//     (b, kv head) merges them with a log-sum-exp (atomic ticket, no waiting);
//   * the last CTA of each (b, kv head) also appends that head's new token to
//     the ring and its queries to the query buffer (every split of the head is
//     done reading by then); the last CTA of the grid advances T;
//   * launched with programmatic dependent launch: a CTA prefetches its split's
//     pages and VL rows into L2 before it waits for the previous grid, and lets
//     the next grid launch as soon as its own wait is over.
#include "common.cuh"

namespace hq {
namespace {

// Two CTA shapes, one kernel template (NC consumer warps, 2 stages each, one
// producer warp):
//   wide  : NC = 11, 22 stages, 1 CTA per SM  (few kv heads: fewer, longer splits)
//   narrow: NC = 3,  6 stages, 3 CTAs per SM  (large batches)
// Each stage must have exactly one consumer warp: a parity wait on an mbarrier
// only tells the current phase from the one before it, so a warp that reached a
// stage while another warp's earlier tile there had not landed yet would see the
// older completed phase and consume the wrong data.  With NSTAGES = 2 NC,
// stage s belongs to warp s % NC.
#ifndef HQ_DECODE_NC_WIDE
#define HQ_DECODE_NC_WIDE 11
#endif
constexpr int NC_WIDE = HQ_DECODE_NC_WIDE, NC_NARROW = 3;
constexpr int PK = 64;                         // positions per packed tile
constexpr int FT = 16;                         // rows per FP16 tile
constexpr int FSTRIDE = 256;                   // bytes per FP16 row in shared memory (one contiguous copy)
constexpr int OFF_VC = 4096, OFF_KS = 8192, OFF_VS = 9216, OFF_MASK = 10240;
constexpr int OFF_FV = FT * FSTRIDE;           // V rows of an FP16 tile
constexpr int STAGE_BYTES = 10368;             // max(10256, 2 * 16 * 256 = 8192), 128-aligned
constexpr int PART_FLOATS = 16 + 8 * D;        // m[8], l[8], O[8][128]
constexpr int MAX_SPLITS = 64;                 // splits per (b, kv head)
constexpr uint32_t PK_TX = HQ_PAGE_VLMASK + 16;   // codes, scale/zero words and the bitmap: one copy
static_assert(OFF_VC == HQ_PAGE_VCODES && OFF_KS == HQ_PAGE_KSZ && OFF_VS == HQ_PAGE_VSZ && OFF_MASK == HQ_PAGE_VLMASK,
              "a packed stage is a verbatim copy of the page prefix");

// key slot -> shared-memory row inside a 16-key block.  Packed tiles (64-byte
// rows): {0,5,1,4,2,7,3,6, 8,13,9,12,10,15,11,14}; FP16 tiles (256-byte rows):
// {0,2,1,3,4,6,5,7, 8,10,9,11,12,14,13,15}.  The packed map keeps the QK rows
// of a quarter-warp and the PV rows of a warp on distinct banks.
__device__ __forceinline__ int pi_pk(int s) {
  const int x = s & 7;
  return (s & 8) + ((x & 1) ? 4 + ((x >> 1) ^ 1) : (x >> 1));
}
__device__ __forceinline__ int pi_fp(int s) {
  const int x = s & 7;
  return (s & 8) + (x & 4) + ((x & 1) << 1) + ((x >> 1) & 1);
}

struct Geo {
  int n_packed, n_vl, T, R, NP, NV, NR, NT;
};

// tiles of one (b, kv head): [0, NP) packed, [NP, NP+NV) VL, [NP+NV, NT-1) ring
// (R/16 slot tiles), NT-1 the new token
__device__ __forceinline__ Geo geo_of(int n_packed, int n_vl, int T, int R) {
  Geo g;
  g.n_packed = n_packed;
  g.n_vl = n_vl;
  g.T = T;
  g.R = R;
  g.NP = (n_packed + PK - 1) / PK;
  g.NV = (n_vl + FT - 1) / FT;
  g.NR = R / FT + 1;
  g.NT = g.NP + g.NV + g.NR;
  return g;
}

// 16-bit mask of the valid rows of FP16 tile `tile`
__device__ __forceinline__ uint32_t fp16_valid(const Geo& g, int tile) {
  if (tile < g.NP + g.NV) {
    const int first = (tile - g.NP) * FT;
    const int n = min(FT, g.n_vl - first);
    return n >= FT ? 0xFFFFu : ((1u << n) - 1u);
  }
  const int j = tile - g.NP - g.NV;
  if (j == g.NR - 1) return 1u;  // the new token
  // ring slot s holds position p = n_packed + ((s - n_packed) mod R); valid iff p < T
  const int base = g.n_packed % g.R;
  uint32_t m = 0;
#pragma unroll 4
  for (int r = 0; r < FT; ++r) {
    int off = FT * j + r - base;
    off += off < 0 ? g.R : 0;
    m |= (g.n_packed + off < g.T ? 1u : 0u) << r;
  }
  return m;
}

// This split's tiles: an even share of the packed tiles [p_lo, p_lo + n_p)
// and an even share of the FP16 tiles [f_lo, f_lo + n_f) (VL, ring, new
// token), numbered 0 .. n_p + n_f - 1 packed first.  Consumer warps take them
// round-robin, so the FP16 tiles (8 KB each, like a packed tile's 10 KB, but
// about a tenth of its arithmetic) land on the warps that got one packed tile
// fewer: the slowest warp of a split does ceil(n_p / NC) packed tiles plus at
// most one FP16 tile, and every split streams about the same bytes.
struct SplitTiles {
  int p_lo, n_p, f_lo, n_f;
  __device__ __forceinline__ int tile(int i) const { return i < n_p ? p_lo + i : f_lo + (i - n_p); }
};
__device__ __forceinline__ SplitTiles split_tiles(const Geo& geo, int split, int S) {
  SplitTiles r;
  const int NF = geo.NT - geo.NP;
  r.p_lo = static_cast<int>((static_cast<long long>(split) * geo.NP) / S);
  r.n_p = static_cast<int>((static_cast<long long>(split + 1) * geo.NP) / S) - r.p_lo;
  const int f0 = static_cast<int>((static_cast<long long>(split) * NF) / S);
  r.f_lo = geo.NP + f0;
  r.n_f = static_cast<int>((static_cast<long long>(split + 1) * NF) / S) - f0;
  return r;
}

struct WarpState {
  float m[2], l[2];
  float o[8][4];
};

// Online-softmax update for NMT 16-key blocks whose S^T accumulators are in s.
// Returns the P^T B-fragments (two per block) in pb.
// Online-softmax update for NMT 16-key blocks whose S^T accumulators are in s.
// Returns the P^T B-fragments (two per block) in pb.  The running max moves
// lazily: only when a query's tile max exceeds it by more than LAZY_MAX (log2
// units), so most tiles skip the rescale of O and l; p then stays below
// 2^LAZY_MAX, well inside fp16, and l accumulates in fp32.
constexpr float LAZY_MAX = 8.0f;

template <int NMT>
__device__ __forceinline__ void softmax_update(WarpState& ws, float (&s)[NMT][4], uint32_t (&pb)[NMT][2]) {
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int i = 0; i < NMT; ++i) {
    mx0 = fmaxf(mx0, fmaxf(s[i][0], s[i][2]));
    mx1 = fmaxf(mx1, fmaxf(s[i][1], s[i][3]));
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  const bool up0 = mx0 > ws.m[0] + LAZY_MAX, up1 = mx1 > ws.m[1] + LAZY_MAX;
  if (__any_sync(0xffffffffu, up0 || up1)) {
    // exp2(-inf) = 0 when the old max is -inf (O and l are still zero then)
    const float c0 = up0 ? ex2(ws.m[0] - mx0) : 1.f, c1 = up1 ? ex2(ws.m[1] - mx1) : 1.f;
    ws.m[0] = up0 ? mx0 : ws.m[0];
    ws.m[1] = up1 ? mx1 : ws.m[1];
    ws.l[0] *= c0;
    ws.l[1] *= c1;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      ws.o[m][0] *= c0;
      ws.o[m][2] *= c0;
      ws.o[m][1] *= c1;
      ws.o[m][3] *= c1;
    }
  }
  const float ref0 = ws.m[0] == -INFINITY ? 0.f : ws.m[0];
  const float ref1 = ws.m[1] == -INFINITY ? 0.f : ws.m[1];
#pragma unroll
  for (int i = 0; i < NMT; ++i) {
    const float p0 = ex2(s[i][0] - ref0), p1 = ex2(s[i][1] - ref1);
    const float p2 = ex2(s[i][2] - ref0), p3 = ex2(s[i][3] - ref1);
    ws.l[0] += p0 + p2;
    ws.l[1] += p1 + p3;
    pb[i][0] = movmatrix_t(pack_f16x2(p0, p1));
    pb[i][1] = movmatrix_t(pack_f16x2(p2, p3));
  }
}

// one K4V4 packed tile (64 positions) by one warp: S^T = K^ . Q^T for the four
// 16-key blocks, one online-softmax step for all 64 keys, O^T += V^T . P^T
__device__ __forceinline__ void packed_tile(WarpState& ws, const uint8_t* st, const uint32_t (&qf)[8][2], int tile, int n_packed,
                                            float qscale, int g, int t) {
  const uint8_t* kc = st;
  const uint8_t* vc = st + OFF_VC;
  const uint32_t* ks = reinterpret_cast<const uint32_t*>(st + OFF_KS);
  const uint32_t* vs = reinterpret_cast<const uint32_t*>(st + OFF_VS);
  const uint32_t* mk = reinterpret_cast<const uint32_t*>(st + OFF_MASK);
  const int base = tile * PK;
  const bool full = base + PK <= n_packed;
  const int pa = pi_pk(g), pbk = pi_pk(g + 8);
  // additive score bias of this thread's 8 key rows: -inf beyond n_packed or on
  // a vertical line (its FP16 row is read instead), else 0
  const uint32_t m0 = mk[0], m1 = mk[1];
  float bias[4][2];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    const uint32_t w = (mt >> 1) ? m1 : m0;
    const int ra = 16 * mt + pa, rb = 16 * mt + pbk;
    const bool va = (full || base + ra < n_packed) && !((w >> (ra & 31)) & 1u);
    const bool vb = (full || base + rb < n_packed) && !((w >> (rb & 31)) & 1u);
    bias[mt][0] = va ? 0.f : -INFINITY;
    bias[mt][1] = vb ? 0.f : -INFINITY;
  }

  float s[4][4];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    const int ra = 16 * mt + pa, rb = 16 * mt + pbk;
    const uint4 ka = *reinterpret_cast<const uint4*>(kc + ra * 64 + 16 * t);
    const uint4 kb = *reinterpret_cast<const uint4*>(kc + rb * 64 + 16 * t);
    const uint32_t za = ks[ra * 4 + t], zb = ks[rb * 4 + t];
    const uint32_t sa2 = prmt(za, za, 0x1010), za2 = prmt(za, za, 0x3232);
    const uint32_t sb2 = prmt(zb, zb, 0x1010), zb2 = prmt(zb, zb, 0x3232);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t wa[4] = {ka.x, ka.y, ka.z, ka.w};
    const uint32_t wb[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t xa = wa[i] >> (8 * h), xb = wb[i] >> (8 * h);
        const uint32_t a0 = hfma2_u(nib_lo(xa), sa2, za2);
        const uint32_t a2 = hfma2_u(nib_hi(xa), sa2, za2);
        const uint32_t a1 = hfma2_u(nib_lo(xb), sb2, zb2);
        const uint32_t a3 = hfma2_u(nib_hi(xb), sb2, zb2);
        mma16816(acc, a0, a1, a2, a3, qf[2 * i + h][0], qf[2 * i + h][1]);
      }
    }
    s[mt][0] = fmaf(acc[0], qscale, bias[mt][0]);
    s[mt][1] = fmaf(acc[1], qscale, bias[mt][0]);
    s[mt][2] = fmaf(acc[2], qscale, bias[mt][1]);
    s[mt][3] = fmaf(acc[3], qscale, bias[mt][1]);
  }
  uint32_t pb[4][2];
  softmax_update<4>(ws, s, pb);

#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    const int r0 = 16 * mt + pi_pk(2 * t), r1 = 16 * mt + pi_pk(2 * t + 1);
    const int r2 = 16 * mt + pi_pk(2 * t + 8), r3 = 16 * mt + pi_pk(2 * t + 9);
    // two 32-bit loads per row, issued in a per-thread order that keeps the
    // warp's accesses on distinct banks
    const int e = t >> 1;
    const uint32_t* v0 = reinterpret_cast<const uint32_t*>(vc + r0 * 64) + 2 * g;
    const uint32_t* v1 = reinterpret_cast<const uint32_t*>(vc + r1 * 64) + 2 * g;
    const uint32_t* v2 = reinterpret_cast<const uint32_t*>(vc + r2 * 64) + 2 * g;
    const uint32_t* v3 = reinterpret_cast<const uint32_t*>(vc + r3 * 64) + 2 * g;
    const uint32_t x0a = v0[e], x0b = v0[e ^ 1], x1a = v1[e], x1b = v1[e ^ 1];
    const uint32_t x2a = v2[e], x2b = v2[e ^ 1], x3a = v3[e], x3b = v3[e ^ 1];
    // un-rotate: w?0 = word 2g, w?1 = word 2g+1
    const uint32_t w00 = e ? x0b : x0a, w01 = e ? x0a : x0b;
    const uint32_t w10 = e ? x1b : x1a, w11 = e ? x1a : x1b;
    const uint32_t w20 = e ? x2b : x2a, w21 = e ? x2a : x2b;
    const uint32_t w30 = e ? x3b : x3a, w31 = e ? x3a : x3b;
    const int grp = g >> 1;
    const uint32_t z0 = vs[r0 * 4 + grp], z1 = vs[r1 * 4 + grp], z2 = vs[r2 * 4 + grp], z3 = vs[r3 * 4 + grp];
    const uint32_t s01 = prmt(z0, z1, 0x5410), o01 = prmt(z0, z1, 0x7632);
    const uint32_t s23 = prmt(z2, z3, 0x5410), o23 = prmt(z2, z3, 0x7632);
    // pair nibbles of the two keys: x?[k] holds dims 16g + 4k .. 16g + 4k + 3 of both keys
    uint32_t xab[4], xcd[4];
    xab[0] = prmt(w00, w10, 0x5410);
    xab[1] = prmt(w00, w10, 0x7632);
    xab[2] = prmt(w01, w11, 0x5410);
    xab[3] = prmt(w01, w11, 0x7632);
    xcd[0] = prmt(w20, w30, 0x5410);
    xcd[1] = prmt(w20, w30, 0x7632);
    xcd[2] = prmt(w21, w31, 0x5410);
    xcd[3] = prmt(w21, w31, 0x7632);
    uint32_t keep_ab = 0xFFFFFFFFu, keep_cd = 0xFFFFFFFFu;
    if (!full) {  // rows past n_packed may hold stale records: zero them out of P.V
      keep_ab = (base + r0 < n_packed ? 0x0000FFFFu : 0u) | (base + r1 < n_packed ? 0xFFFF0000u : 0u);
      keep_cd = (base + r2 < n_packed ? 0x0000FFFFu : 0u) | (base + r3 < n_packed ? 0xFFFF0000u : 0u);
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const uint32_t yab = xab[m >> 1] >> (8 * (m & 1));
      const uint32_t ycd = xcd[m >> 1] >> (8 * (m & 1));
      uint32_t a0 = hfma2_u(nib_lo(yab), s01, o01);
      uint32_t a1 = hfma2_u(nib_hi(yab), s01, o01);
      uint32_t a2 = hfma2_u(nib_lo(ycd), s23, o23);
      uint32_t a3 = hfma2_u(nib_hi(ycd), s23, o23);
      if (!full) {
        a0 &= keep_ab; a1 &= keep_ab;
        a2 &= keep_cd; a3 &= keep_cd;
      }
      mma16816(ws.o[m], a0, a1, a2, a3, pb[mt][0], pb[mt][1]);
    }
  }
}

// one FP16 tile (16 rows at FSTRIDE) by one warp; bit r of `valid` marks row r as real
__device__ __forceinline__ void fp16_tile(WarpState& ws, const uint8_t* st, const uint32_t (&qf)[8][2], uint32_t valid,
                                          float qscale, int g, int t) {
  const uint8_t* kb = st;
  const uint8_t* vb = st + OFF_FV;
  const int ra = pi_fp(g), rb = pi_fp(g + 8);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 ua = *reinterpret_cast<const uint4*>(kb + ra * FSTRIDE + 64 * t + 16 * i);
    const uint4 ub = *reinterpret_cast<const uint4*>(kb + rb * FSTRIDE + 64 * t + 16 * i);
    // k-step 2i: (d0,d4) and (d1,d5); k-step 2i+1: (d2,d6) and (d3,d7)
    mma16816(acc, prmt(ua.x, ua.z, 0x5410), prmt(ub.x, ub.z, 0x5410), prmt(ua.x, ua.z, 0x7632), prmt(ub.x, ub.z, 0x7632),
             qf[2 * i][0], qf[2 * i][1]);
    mma16816(acc, prmt(ua.y, ua.w, 0x5410), prmt(ub.y, ub.w, 0x5410), prmt(ua.y, ua.w, 0x7632), prmt(ub.y, ub.w, 0x7632),
             qf[2 * i + 1][0], qf[2 * i + 1][1]);
  }
  float s[1][4];
  const bool va = (valid >> ra) & 1u, vbv = (valid >> rb) & 1u;
  s[0][0] = va ? acc[0] * qscale : -INFINITY;
  s[0][1] = va ? acc[1] * qscale : -INFINITY;
  s[0][2] = vbv ? acc[2] * qscale : -INFINITY;
  s[0][3] = vbv ? acc[3] * qscale : -INFINITY;
  uint32_t pb[1][2];
  softmax_update<1>(ws, s, pb);

  const int r0 = pi_fp(2 * t), r1 = pi_fp(2 * t + 1), r2 = pi_fp(2 * t + 8), r3 = pi_fp(2 * t + 9);
  const uint4 a0l = *reinterpret_cast<const uint4*>(vb + r0 * FSTRIDE + 32 * g);
  const uint4 a0h = *reinterpret_cast<const uint4*>(vb + r0 * FSTRIDE + 32 * g + 16);
  const uint4 a1l = *reinterpret_cast<const uint4*>(vb + r1 * FSTRIDE + 32 * g);
  const uint4 a1h = *reinterpret_cast<const uint4*>(vb + r1 * FSTRIDE + 32 * g + 16);
  const uint4 a2l = *reinterpret_cast<const uint4*>(vb + r2 * FSTRIDE + 32 * g);
  const uint4 a2h = *reinterpret_cast<const uint4*>(vb + r2 * FSTRIDE + 32 * g + 16);
  const uint4 a3l = *reinterpret_cast<const uint4*>(vb + r3 * FSTRIDE + 32 * g);
  const uint4 a3h = *reinterpret_cast<const uint4*>(vb + r3 * FSTRIDE + 32 * g + 16);
  uint32_t w0[8] = {a0l.x, a0l.y, a0l.z, a0l.w, a0h.x, a0h.y, a0h.z, a0h.w};
  uint32_t w1[8] = {a1l.x, a1l.y, a1l.z, a1l.w, a1h.x, a1h.y, a1h.z, a1h.w};
  uint32_t w2[8] = {a2l.x, a2l.y, a2l.z, a2l.w, a2h.x, a2h.y, a2h.z, a2h.w};
  uint32_t w3[8] = {a3l.x, a3l.y, a3l.z, a3l.w, a3h.x, a3h.y, a3h.z, a3h.w};
  if (valid != 0xFFFFu) {  // invalid rows may hold stale bytes: keep them out of P.V
    const uint32_t k0 = ((valid >> r0) & 1u) ? 0xFFFFFFFFu : 0u, k1 = ((valid >> r1) & 1u) ? 0xFFFFFFFFu : 0u;
    const uint32_t k2 = ((valid >> r2) & 1u) ? 0xFFFFFFFFu : 0u, k3 = ((valid >> r3) & 1u) ? 0xFFFFFFFFu : 0u;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      w0[m] &= k0; w1[m] &= k1; w2[m] &= k2; w3[m] &= k3;
    }
  }
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    mma16816(ws.o[m], prmt(w0[m], w1[m], 0x5410), prmt(w0[m], w1[m], 0x7632), prmt(w2[m], w3[m], 0x5410),
             prmt(w2[m], w3[m], 0x7632), pb[0][0], pb[0][1]);
  }
}

template <int NCONS, int MINB>
__global__ void __launch_bounds__((NCONS + 1) * 32, MINB)
decode_kernel(const hq_cache c, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k_new,
              const uint16_t* __restrict__ v_new, uint16_t* __restrict__ out, float qscale, int S,
              float* __restrict__ parts, unsigned int* __restrict__ tickets) {
  constexpr int NSTAGES = 2 * NCONS;
  constexpr int NTHREADS = (NCONS + 1) * 32;
  static_assert(NSTAGES % NCONS == 0, "every stage needs a single owner warp");
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[NSTAGES], empty[NSTAGES];
  __shared__ int s_last;
  __shared__ int s_timeout;      // a bounded wait gave up somewhere in this CTA
  __shared__ int s_issued[NSTAGES];  // tiles issued into each stage

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int bh = b * c.Hkv + kvh;
  const int G = c.Hq / c.Hkv;
  const int R = ring_len(c.W);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      s_issued[i] = 0;
    }
    s_timeout = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == NCONS * 32) {
    // Before the dependency wait, warm L2 with this split's packed pages and VL
    // rows.  The lengths read here may be stale (the previous grid can still be
    // writing them): they only steer a prefetch hint, and the ranges are clamped
    // to the buffers, so a stale value costs bandwidth, never correctness.
    const int pT = *reinterpret_cast<volatile const int*>(c.state + HQ_STATE_T);
    const int pnp = *reinterpret_cast<volatile const int*>(c.state + HQ_STATE_NPACKED);
    const int pnv = *reinterpret_cast<volatile const int*>(c.state + HQ_STATE_NVL);
    const Geo pg = geo_of(min(max(pnp, 0), c.cap), min(max(pnv, 0), c.vl_cap), pT, R);
    const SplitTiles pr = split_tiles(pg, split, S);
    const int npg = c.cap / PK;
    const int a0 = min(max(pr.p_lo, 0), npg), a1 = min(max(pr.p_lo + pr.n_p, a0), npg);
    const uint8_t* pages = c.pages + static_cast<size_t>(bh) * npg * HQ_PAGE_BYTES;
    for (int pgi = a0; pgi < a1; pgi += 16)  // 16 pages (165 KB) per prefetch
      prefetch_l2(pages + static_cast<size_t>(pgi) * HQ_PAGE_BYTES, min(16, a1 - pgi) * HQ_PAGE_BYTES);
    const int v0 = min(max(pr.f_lo - pg.NP, 0), c.vl_cap / FT);
    const int v1 = min(max(pr.f_lo + pr.n_f - pg.NP, v0), min(pg.NV, c.vl_cap / FT));
    if (v1 > v0) {
      const size_t off = (static_cast<size_t>(bh) * c.vl_cap + v0 * FT) * D;
      prefetch_l2(c.kf + off, (v1 - v0) * FT * D * 2);
      prefetch_l2(c.vf + off, (v1 - v0) * FT * D * 2);
    }
  }
  // programmatic dependent launch: everything this kernel reads (the state, the
  // cache, the previous step's appended token) was written by earlier kernels,
  // so wait for them first; then let the next step's grid start launching onto
  // the SMs that free up (it waits here in turn)
  griddep_wait();
  griddep_launch_dependents();
  const int T = c.state[HQ_STATE_T];
  const int n_packed = c.state[HQ_STATE_NPACKED];
  const int n_vl = c.state[HQ_STATE_NVL];
  if (T - n_packed >= c.W + HQ_STAGE || T >= c.cap) {  // staging full / no room: do nothing
    if (split == 0 && kvh == 0 && b == 0 && threadIdx.x == 0)
      set_err(c.state, T >= c.cap ? HQ_DEVERR_CAPACITY : HQ_DEVERR_STAGING_FULL);
    return;
  }
  const Geo geo = geo_of(n_packed, n_vl, T, R);
  const SplitTiles sp = split_tiles(geo, split, S);
  const int ntile = sp.n_p + sp.n_f;

  __syncthreads();

  WarpState ws;
  ws.m[0] = ws.m[1] = -INFINITY;
  ws.l[0] = ws.l[1] = 0.f;
#pragma unroll
  for (int m = 0; m < 8; ++m) ws.o[m][0] = ws.o[m][1] = ws.o[m][2] = ws.o[m][3] = 0.f;

  if (warp == NCONS) {
    // ---------------------------------------------------------------- producer
    // lane s owns stage s and issues tiles s, s + NSTAGES, s + 2 NSTAGES, ...
    // (1 bulk copy per packed page, 2 per FP16 tile): the initial fill of every
    // stage leaves in one instruction, and a refill waits only for its own stage
    static_assert(NSTAGES <= 32, "one producer lane per stage");
    if (lane < NSTAGES) {
      const int s = lane;
      const size_t npg = static_cast<size_t>(c.cap / PK);
      const uint8_t* pages = c.pages + static_cast<size_t>(bh) * npg * HQ_PAGE_BYTES;
      const uint16_t* kf = c.kf + static_cast<size_t>(bh) * c.vl_cap * D;
      const uint16_t* vf = c.vf + static_cast<size_t>(bh) * c.vl_cap * D;
      const uint16_t* kr = c.kr + static_cast<size_t>(bh) * R * D;
      const uint16_t* vr = c.vr + static_cast<size_t>(bh) * R * D;
      uint8_t* st = smem + s * STAGE_BYTES;
      int k = 0;  // uses of this stage so far
      for (int i = s; i < ntile; i += NSTAGES, ++k) {
        // the k-th refill waits for the consumer's k-th release (phase k - 1)
        if (k > 0 && !mbar_wait(&empty[s], (k - 1) & 1, c.state)) {
          s_timeout = 1;
          break;
        }
        s_issued[s] = k + 1;
        const int tile = sp.tile(i);
        if (tile < geo.NP) {
          mbar_arrive_expect_tx(&full[s], PK_TX);
          bulk_g2s(st, pages + static_cast<size_t>(tile) * HQ_PAGE_BYTES, PK_TX, &full[s]);
        } else {
          const int v = tile - geo.NP, j = v - geo.NV;
          const uint16_t* ksrc = j < 0 ? kf + v * (FT * D) : (j < geo.NR - 1 ? kr + j * (FT * D) : k_new + bh * D);
          const uint16_t* vsrc = j < 0 ? vf + v * (FT * D) : (j < geo.NR - 1 ? vr + j * (FT * D) : v_new + bh * D);
          const uint32_t bytes = j == geo.NR - 1 ? 2 * D : FT * 2 * D;
          mbar_arrive_expect_tx(&full[s], 2 * bytes);
          bulk_g2s(st, ksrc, bytes, &full[s]);
          bulk_g2s(st + OFF_FV, vsrc, bytes, &full[s]);
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- consumers
    // Q^T fragments in the permuted dim order (thread t covers dims 32t .. 32t+31)
    uint32_t qf[8][2];
    if (g < G) {
      const uint4* qp = reinterpret_cast<const uint4*>(q + (static_cast<size_t>(b) * c.Hq + kvh * G + g) * D + 32 * t);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 u = qp[i];
        qf[2 * i][0] = prmt(u.x, u.z, 0x5410);
        qf[2 * i][1] = prmt(u.x, u.z, 0x7632);
        qf[2 * i + 1][0] = prmt(u.y, u.w, 0x5410);
        qf[2 * i + 1][1] = prmt(u.y, u.w, 0x7632);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) qf[j][0] = qf[j][1] = 0u;
    }
    for (int i = warp; i < ntile; i += NCONS) {
      const int s = i % NSTAGES;
      // the timeout decision is made warp-uniform so the warp never splits
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (i / NSTAGES) & 1, c.state))) {
        if (lane == 0) s_timeout = 1;
        break;
      }
      const uint8_t* st = smem + s * STAGE_BYTES;
      const int tile = sp.tile(i);
      if (tile < geo.NP) {
        packed_tile(ws, st, qf, tile, n_packed, qscale, g, t);
      } else {
        fp16_tile(ws, st, qf, fp16_valid(geo, tile), qscale, g, t);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // l: sum the per-thread partial sums over the 8 lanes of a query column
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      ws.l[0] += __shfl_xor_sync(0xffffffffu, ws.l[0], o);
      ws.l[1] += __shfl_xor_sync(0xffffffffu, ws.l[1], o);
    }
  }
  __syncthreads();  // (A) every tile consumed: stage memory is free for the merge
  if (s_timeout) {
    // never expected: before the stage memory is reused or the CTA exits, wait
    // (bounded) for every bulk copy this CTA issued to land
    if (threadIdx.x == 0)
      for (int st = 0; st < NSTAGES; ++st)
        if (s_issued[st] > 0) mbar_wait(&full[st], (s_issued[st] - 1) & 1, c.state);
    __syncthreads();
  }
  if (warp < NCONS) {
    float* wsm = reinterpret_cast<float*>(smem) + warp * PART_FLOATS;
    if (g == 0) {
      wsm[2 * t] = ws.m[0];
      wsm[2 * t + 1] = ws.m[1];
      wsm[8 + 2 * t] = ws.l[0];
      wsm[8 + 2 * t + 1] = ws.l[1];
    }
    float* wo = wsm + 16;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      wo[(2 * t) * D + 16 * g + 2 * m] = ws.o[m][0];
      wo[(2 * t + 1) * D + 16 * g + 2 * m] = ws.o[m][1];
      wo[(2 * t) * D + 16 * g + 2 * m + 1] = ws.o[m][2];
      wo[(2 * t + 1) * D + 16 * g + 2 * m + 1] = ws.o[m][3];
    }
  }
  __syncthreads();  // (B) warp states visible

  // ---------------------------------------------------------------- CTA merge -> split partial
  // each thread owns 4 dims of one query and weighs the NC warp states itself
  // (NC exp2 per thread instead of a third barrier)
  __shared__ int s_glast;
  const float* wsm = reinterpret_cast<const float*>(smem);
  float* part = parts + (static_cast<size_t>(bh) * S + split) * PART_FLOATS;
  for (int i = threadIdx.x; i < 8 * D / 4; i += NTHREADS) {
    const int qc = (4 * i) / D;
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < NCONS; ++w) mm = fmaxf(mm, wsm[w * PART_FLOATS + qc]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float ll = 0.f;
#pragma unroll
    for (int w = 0; w < NCONS; ++w) {
      const float mw = wsm[w * PART_FLOATS + qc];
      const float wt = mw == -INFINITY ? 0.f : ex2(mw - mm);
      const float4 o = reinterpret_cast<const float4*>(wsm + w * PART_FLOATS + 16)[i];
      acc.x = fmaf(wt, o.x, acc.x);
      acc.y = fmaf(wt, o.y, acc.y);
      acc.z = fmaf(wt, o.z, acc.z);
      acc.w = fmaf(wt, o.w, acc.w);
      ll = fmaf(wt, wsm[w * PART_FLOATS + 8 + qc], ll);
    }
    reinterpret_cast<float4*>(part + 16)[i] = acc;
    if ((4 * i) % D == 0) {
      part[qc] = mm;
      part[8 + qc] = ll;
    }
  }
  // the new token's K / V rows and this group's queries, loaded now so that the
  // append after the ticket is stores only (inputs: no ordering concerns)
  const int slot = T % R;
  constexpr int APPEND_MAX = (2 + HQ_MAX_GQA) * (D / 8);
  static_assert(APPEND_MAX <= 2 * NTHREADS, "at most two 16-byte chunks of the append per thread");
  uint4 app[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
  uint4* app_dst[2] = {nullptr, nullptr};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int e = threadIdx.x + k * NTHREADS;
    if (e < (2 + G) * (D / 8)) {
      const int row = e / (D / 8), ch = e % (D / 8);
      if (row < 2) {
        app[k] = reinterpret_cast<const uint4*>((row ? v_new : k_new) + static_cast<size_t>(bh) * D)[ch];
        app_dst[k] = reinterpret_cast<uint4*>((row ? c.vr : c.kr) + (static_cast<size_t>(bh) * R + slot) * D) + ch;
      } else {
        const size_t h = static_cast<size_t>(b) * c.Hq + kvh * G + (row - 2);
        app[k] = reinterpret_cast<const uint4*>(q + h * D)[ch];
        app_dst[k] = reinterpret_cast<uint4*>(c.qbuf + (h * HQ_QBUF + (T % HQ_QBUF)) * D) + ch;
      }
    }
  }
  // completion tickets: the barrier orders every thread's partial writes before
  // thread 0's gpu-scope release; the two counters are bumped together; the
  // last CTA of the head (and/or of the grid) acquires before the barrier that
  // releases its other threads to read the partials
  __syncthreads();
  if (threadIdx.x == 0) {
    fence_acq_rel_gpu();
    const unsigned int th = atomicAdd(&tickets[1 + bh], 1u);
    const unsigned int tg = atomicAdd(&tickets[0], 1u);
    s_last = th == static_cast<unsigned>(S - 1);
    s_glast = tg == gridDim.x * gridDim.y * gridDim.z - 1;
    if (s_last || s_glast) fence_acq_rel_gpu();
  }
  __syncthreads();
  if (s_last) {
    // log-sum-exp merge of the S partials of this (b, kv head).  The threads
    // split into ngrp groups, each summing the O partials of every ngrp-th split
    // for one (query, 4 dims) item; a thread's first PER O loads are issued
    // before the (m, l) of the splits are gathered and weighed, so both round
    // trips to L2 overlap, and the groups' sums meet in shared memory.
    const float* pb = parts + static_cast<size_t>(bh) * S * PART_FLOATS;
    float* sm_m = reinterpret_cast<float*>(smem);      // [S][8]: the split weights
    float* sm_inv = sm_m + 2 * 64 * 8;                  // [8]
    float4* red = reinterpret_cast<float4*>(sm_inv + 8);  // [ngrp][items]
    constexpr int PER = 8;
    const int items = G * (D / 4);
    const bool grouped = items <= NTHREADS;             // else one pass over items per thread stride
    const int ngrp = grouped ? max(1, min(NTHREADS / items, S)) : 1;
    const int grp = grouped ? threadIdx.x / items : 0;
    const int it0 = threadIdx.x - grp * items;
    const bool mine = grouped && grp < ngrp;
    const float4* osrc = reinterpret_cast<const float4*>(pb + 16 + (it0 / (D / 4)) * D) + it0 % (D / 4);
    float4 ov[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int sp = grp + j * ngrp;
      ov[j] = (mine && sp < S) ? __ldcg(osrc + sp * (PART_FLOATS / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // split weights: warp qc weighs query qc's splits, lane s holding splits s
    // and s + 32 (S <= 64), with warp-wide max and sum
    static_assert(MAX_SPLITS <= 64, "two splits per lane");
    for (int qc = warp; qc < G; qc += NTHREADS / 32) {
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
      if (lane < S) {
        m0 = __ldcg(pb + lane * PART_FLOATS + qc);
        l0 = __ldcg(pb + lane * PART_FLOATS + 8 + qc);
      }
      if (lane + 32 < S) {
        m1 = __ldcg(pb + (lane + 32) * PART_FLOATS + qc);
        l1 = __ldcg(pb + (lane + 32) * PART_FLOATS + 8 + qc);
      }
      float mm = fmaxf(m0, m1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, o));
      const float w0 = m0 == -INFINITY ? 0.f : ex2(m0 - mm);
      const float w1 = m1 == -INFINITY ? 0.f : ex2(m1 - mm);
      float ll = w0 * l0 + w1 * l1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ll += __shfl_xor_sync(0xffffffffu, ll, o);
      if (lane < S) sm_m[lane * 8 + qc] = w0;
      if (lane + 32 < S) sm_m[(lane + 32) * 8 + qc] = w1;
      if (lane == 0) sm_inv[qc] = ll > 0.f ? 1.0f / ll : 0.f;
    }
    __syncthreads();
    auto store_out = [&](int it, const float4& acc) {
      const int qc = it / (D / 4), d4 = it % (D / 4);
      const float inv = sm_inv[qc];
      __half2* dst = reinterpret_cast<__half2*>(out + (static_cast<size_t>(b) * c.Hq + kvh * G + qc) * D) + 2 * d4;
      dst[0] = __floats2half2_rn(acc.x * inv, acc.y * inv);
      dst[1] = __floats2half2_rn(acc.z * inv, acc.w * inv);
    };
    if (grouped) {
      if (mine) {
        const int qc = it0 / (D / 4);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < PER; ++j) {
          const int sp = grp + j * ngrp;
          const float w = sp < S ? sm_m[sp * 8 + qc] : 0.f;
          acc.x = fmaf(w, ov[j].x, acc.x);
          acc.y = fmaf(w, ov[j].y, acc.y);
          acc.z = fmaf(w, ov[j].z, acc.z);
          acc.w = fmaf(w, ov[j].w, acc.w);
        }
        for (int sp = grp + PER * ngrp; sp < S; sp += ngrp) {  // more than PER splits per group
          const float4 o = __ldcg(osrc + sp * (PART_FLOATS / 4));
          const float w = sm_m[sp * 8 + qc];
          acc.x = fmaf(w, o.x, acc.x);
          acc.y = fmaf(w, o.y, acc.y);
          acc.z = fmaf(w, o.z, acc.z);
          acc.w = fmaf(w, o.w, acc.w);
        }
        red[grp * items + it0] = acc;
      }
      __syncthreads();
      if (threadIdx.x < items) {
        float4 acc = red[threadIdx.x];
        for (int g2 = 1; g2 < ngrp; ++g2) {
          const float4 o = red[g2 * items + threadIdx.x];
          acc.x += o.x;
          acc.y += o.y;
          acc.z += o.z;
          acc.w += o.w;
        }
        store_out(threadIdx.x, acc);
      }
    } else {
      for (int it = threadIdx.x; it < items; it += NTHREADS) {
        const int qc = it / (D / 4), d4 = it % (D / 4);
        const float4* src = reinterpret_cast<const float4*>(pb + 16 + qc * D) + d4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int sp = 0; sp < S; ++sp) {
          const float4 o = __ldcg(src + sp * (PART_FLOATS / 4));
          const float w = sm_m[sp * 8 + qc];
          acc.x = fmaf(w, o.x, acc.x);
          acc.y = fmaf(w, o.y, acc.y);
          acc.z = fmaf(w, o.z, acc.z);
          acc.w = fmaf(w, o.w, acc.w);
        }
        store_out(it, acc);
      }
    }
    // every split of this head has consumed its tiles: append the new token to
    // the ring (slot T % R) and this group's queries to the query buffer
    if (app_dst[0]) *app_dst[0] = app[0];
    if (app_dst[1]) *app_dst[1] = app[1];
    if (threadIdx.x == 0) tickets[1 + bh] = 0u;
  }
  // the last CTA of the grid advances T (every CTA read the state at its start)
  if (s_glast && threadIdx.x == 0) {
    c.state[HQ_STATE_T] = T + 1;
    c.state[HQ_STATE_NQ] = min(c.state[HQ_STATE_NQ] + 1, HQ_QBUF);
    tickets[0] = 0u;
  }
}

}  // namespace

// Launch shape: the wide CTA (one per SM) when every (b, kv head) can get at
// least 4 of them, else 3 narrow CTAs per SM; never more than one wave.
struct DecodeShape {
  int S;      // splits per (b, kv head)
  bool wide;
};

DecodeShape decode_shape(const hq_cache& c, int sms) {
  const int units = c.B * c.Hkv;
  const int nt_max = c.cap / PK + c.vl_cap / FT + ring_len(c.W) / FT + 1;
  DecodeShape d;
  d.wide = sms / units >= 4;
  int s = d.wide ? sms / units : (3 * sms) / units;
  const int cap_s = d.wide ? (nt_max + NC_WIDE - 1) / NC_WIDE : (nt_max + NC_NARROW - 1) / NC_NARROW;  // ~one tile per consumer warp
  if (s > cap_s) s = cap_s;
  if (s > MAX_SPLITS) s = MAX_SPLITS;
  if (s < 1) s = 1;
  d.S = s;
  return d;
}

int decode_splits(const hq_cache& c, int sms) { return decode_shape(c, sms).S; }

// counters: [0] grid ticket, [1 + b*Hkv + h] split tickets; zero between calls
size_t decode_counter_bytes(const hq_cache& c) { return ((4ull * (1 + c.B * c.Hkv) + 255) / 256) * 256; }

size_t decode_workspace(const hq_cache& c, int sms) {
  const int S = decode_splits(c, sms);
  return decode_counter_bytes(c) + static_cast<size_t>(c.B) * c.Hkv * S * PART_FLOATS * sizeof(float);
}

hq_status launch_decode(const hq_cache& c, const uint16_t* q, const uint16_t* kn, const uint16_t* vn, uint16_t* out,
                        float sm_scale, void* ws, int sms, cudaStream_t st) {
  const DecodeShape shp = decode_shape(c, sms);
  const int nc = shp.wide ? NC_WIDE : NC_NARROW;
  const int smem = 2 * nc * STAGE_BYTES;
  int dev = 0;
  cudaGetDevice(&dev);
  static DeviceOnce attrs;
  const cudaError_t ea = attrs.run(dev, [] {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<NC_WIDE, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         2 * NC_WIDE * STAGE_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_kernel<NC_NARROW, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               2 * NC_NARROW * STAGE_BYTES);
    return e;
  });
  if (ea != cudaSuccess) return cuda_fail(ea, "decode attributes");
  unsigned int* tickets = reinterpret_cast<unsigned int*>(ws);
  float* parts = reinterpret_cast<float*>(static_cast<char*>(ws) + decode_counter_bytes(c));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(shp.S, c.Hkv, c.B);
  cfg.blockDim = dim3((nc + 1) * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float qs = sm_scale * LOG2E;
  const cudaError_t e = shp.wide
      ? cudaLaunchKernelEx(&cfg, decode_kernel<NC_WIDE, 1>, c, q, kn, vn, out, qs, shp.S, parts, tickets)
      : cudaLaunchKernelEx(&cfg, decode_kernel<NC_NARROW, 3>, c, q, kn, vn, out, qs, shp.S, parts, tickets);
  return cuda_status(e, "decode launch");
}

}  // namespace hq
