// select.cu — vertical-line selection: column-mass scores + exact top-k.
//
// HyQuant digest (agihunt.info), method paragraph; README Overview item 1:
// the vertical-line score of a key is the accumulated column-direction
// attention mass, measured from at most 64 buffered FP16 queries; the top-rho
// of the non-window prefix is kept FP16; reselection runs every 64 tokens.
//
// score_j = sum over the group's query heads h and buffered queries i of
//           softmax_{j' <= p_i}(q_{h,i} . k_j' * sm_scale)[j],   j < n = T - W.
//
// Both passes run on the tcgen05 tensor cores, one CTA per (key range, b, kv
// head), all M = G x nq queries of the group in shared memory:
//   sel_pass<false>  S = Q . K^T (M rows of 128 queries, N = 128 keys) into
//                    TMEM; per query row a running max / sum in the exp2
//                    domain over the CTA's keys -> (m, l) partial per row
//   sel_pass<true>   per-row log-sum-exp from the partials, then
//                    S^T = K . Q^T (M = 128 keys, N = the queries) into TMEM;
//                    per key (one TMEM lane per thread) the sum over queries of
//                    exp2(s - lse) -> score_j, and a histogram of the scores'
//                    bits 30..20 (scores are >= 0, so the bit order is the value
//                    order).  Each key's score is finished inside one CTA.
//   topk             a cluster of 8 CTAs per (b, kv head), each over an eighth
//                    of the positions (one CTA when a range would not fit its
//                    shared memory): the bin holding the k-th largest score from
//                    the histogram, the bin's scores gathered, two 10-bit radix
//                    passes over their low 20 bits (histograms summed across the
//                    cluster) -> the exact k-th value, then an ordered compaction
//                    writes the chosen positions ascending, ties to the lowest
//                    positions
// When the decode steps kept their log-sum-exps (c.qlse) and every buffered
// query came after the last merge, pass 0 is skipped: those are its row sums.
// With running scores (c.score_acc), pass 1 adds each key's column mass to its
// stored sum (decode mode) or starts it (init mode) and ranks the sums.
// Keys are rebuilt as fp16 in their current representation (dense prefix in
// init mode; ring, VL row or dequantised K4V4 record in decode mode) by four
// builder warps straight into the 128-byte-swizzled K-major operand layout.
// Warp roles (416 threads): warps 0-7 epilogue (column half = warp / 4, TMEM
// lane quarter = warp % 4), warps 8-11 key builders (one key row per thread),
// warp 12 TMEM allocation and the MMA issue.  Every mbarrier wait is bounded
// (about 1 s); a timeout sets HQ_DEVERR_TIMEOUT and the CTA drains its MMAs
// before releasing TMEM.
#include <cooperative_groups.h>

#include "tc.cuh"

namespace hq {
namespace {

constexpr int KT = 128;                  // keys per tile
constexpr int EPI_WARPS = 8;
constexpr int BLD_WARPS = 4;
constexpr int MMA_WARP = EPI_WARPS + BLD_WARPS;
constexpr int SEL_THREADS = (MMA_WARP + 1) * 32;
constexpr int MAX_SPLITS = 32;           // CTAs per (b, kv head)
constexpr int KSTAGE = KT * 256;         // one rebuilt key tile: 2 halves x [128 rows][128 B]
constexpr uint32_t TMEM_COLS = 512;
constexpr int HBINS = 2048;              // score histogram: bits 30..20 of the (non-negative) fp32 pattern

struct SelArgs {
  hq_cache c;
  const uint16_t* k_dense;  // init mode: [B, Hkv, L, D]
  const uint16_t* q_ext;    // init mode: [B, Hq, nq, D]
  int L;                    // init mode length
  int nq_init;
  float* lse_part;          // [B*Hkv][MAX_SPLITS][Mp] x (m, l)
  float* scores;            // [B*Hkv][cap]
  uint32_t* hist;           // [B*Hkv][HBINS] histogram of the scores' bits 30..20
  int S;                    // CTAs per (b, kv head)
  int Mp;                   // query rows in shared memory: G * HQ_QBUF rounded up to 128
  float qscale;             // sm_scale * log2(e)
};

struct SelGeo {
  int T, n, nq, qpos0, n_packed, n_vl;
};

__device__ __forceinline__ SelGeo sel_geo(const SelArgs& a, int b) {
  SelGeo g;
  if (a.k_dense) {
    g.T = a.L;
    g.nq = a.nq_init;
    g.n_packed = 0;
    g.n_vl = 0;
  } else {
    const int32_t* st = state_row(a.c, b);
    g.T = st[HQ_STATE_T];
    g.nq = min(st[HQ_STATE_NQ], HQ_QBUF);
    g.n_packed = st[HQ_STATE_NPACKED];
    g.n_vl = st[HQ_STATE_NVL];
  }
  g.n = max(g.T - a.c.W, 0);
  g.qpos0 = g.T - g.nq;
  return g;
}

__device__ __forceinline__ bool sel_wait(uint64_t* bar, uint32_t parity, int32_t* state, int* abort_flag) {
  if (*reinterpret_cast<volatile int*>(abort_flag)) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile int*>(abort_flag)) return false;
    if (global_ns() - t0 > 1000000000ull) {
      set_err(state, HQ_DEVERR_TIMEOUT);
      *reinterpret_cast<volatile int*>(abort_flag) = 1;
      return false;
    }
  }
}

// 16-byte chunk `ch` (dims 8 ch .. 8 ch + 7) of row `r` in the 128-byte-swizzled
// K-major layout of a tile whose halves (dims 0-63, 64-127) are `half_bytes` apart
__device__ __forceinline__ uint32_t sw128_off(int r, int ch, int half_bytes) {
  return (ch >> 3) * half_bytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
}

// A key row fetched ahead of its conversion.  Rows below n_packed bring their
// 64 code bytes, (scale, zero) words, the page's bitmap word and first-VL row
// into registers with independent loads (no branch on the bitmap before they
// are issued); FP16 rows (dense prefix, ring) record their source, which is
// warmed in L2 and copied to shared memory with cp.async when stored.  A
// vertical line's FP16 row is found from the bitmap once the loads are back.
struct KeyRow {
  const uint4* src;  // FP16 source row, or null
  uint4 code[8];     // 16 * bits code bytes (bits = 4: code[0..3], 8: code[0..7], 2: code[0..1])
  uint4 sz;
  uint2 mask;       // the page's bitmap words
  int vlbase;        // VL-store row of the page's first vertical line
  int j;             // position
  bool packed;
};

__device__ __forceinline__ KeyRow fetch_key_row(const SelArgs& a, const SelGeo& g, int bh, int j) {
  const hq_cache& c = a.c;
  KeyRow k;
  k.src = nullptr;
  k.packed = false;
  k.mask = make_uint2(0u, 0u);
  k.vlbase = 0;
  k.j = j;
  if (j >= g.T) return k;
  if (a.k_dense) {
    k.src = reinterpret_cast<const uint4*>(a.k_dense + (static_cast<size_t>(bh) * a.L + j) * D);
  } else if (j >= g.n_packed) {
    k.src = reinterpret_cast<const uint4*>(c.kr + (static_cast<size_t>(bh) * ring_len(c.W) + (j % ring_len(c.W))) * D);
  } else {
    const PageGeo pg = page_geo(c);
    uint8_t* page = page_of(c, bh, j);
    const uint4* codes = reinterpret_cast<const uint4*>(row_codes(pg, page, 0, j));
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i < pg.kb) k.code[i] = codes[i];
    k.sz = *reinterpret_cast<const uint4*>(row_sz(pg, page, 0, j));
    k.mask = *reinterpret_cast<const uint2*>(page_mask(pg, page));
    k.vlbase = *page_vlbase(pg, page);
    k.packed = true;
  }
  if (k.src) prefetch_l2(k.src, D * 2);
  return k;
}

// Source of a fetched row that must be copied as FP16 (a vertical line of a
// packed page, or a dense / ring row); null for a row to dequantise or zero.
__device__ __forceinline__ const uint4* key_row_src(const SelArgs& a, int bh, const KeyRow& k) {
  if (!k.packed) return k.src;
  const bool hi = (k.j & 63) >= 32;
  const uint32_t w = hi ? k.mask.y : k.mask.x;
  if (!((w >> (k.j & 31)) & 1u)) return nullptr;
  const int below = __popc(w & ((1u << (k.j & 31)) - 1u)) + (hi ? __popc(k.mask.x) : 0);
  return reinterpret_cast<const uint4*>(a.c.kf + (static_cast<size_t>(bh) * a.c.vl_cap + k.vlbase + below) * D);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Write a fetched key row as fp16 into row r of a key stage (FP16 sources by
// cp.async: the caller waits for them before publishing the stage).
__device__ __forceinline__ void store_key_row(const SelArgs& a, int bh, const KeyRow& k, uint8_t* stage, int r) {
  const uint4* src = key_row_src(a, bh, k);
  if (src) {
#pragma unroll
    for (int ch = 0; ch < 16; ++ch) cp_async16(stage + sw128_off(r, ch, KT * 128), src + ch);
    return;
  }
  if (k.packed && kbits_of(a.c) != 4) {
    // 8- or 2-bit codes: each 8-dim chunk from its codes, fp16(zero + q * scale) by one fma
    const int kb = kbits_of(a.c);
    const uint32_t szw[4] = {k.sz.x, k.sz.y, k.sz.z, k.sz.w};
#pragma unroll
    for (int ch = 0; ch < 16; ++ch) {
      const uint32_t s2 = prmt(szw[ch >> 2], szw[ch >> 2], 0x1010), z2 = prmt(szw[ch >> 2], szw[ch >> 2], 0x3232);
      uint32_t h[4];
      if (kb == 8) {  // 8 bytes: words 2 ch, 2 ch + 1 of the 128 code bytes
        const uint4 cw = k.code[ch >> 1];
        const uint32_t w0 = (ch & 1) ? cw.z : cw.x, w1 = (ch & 1) ? cw.w : cw.y;
        h[0] = prmt(w0, 0x64646464u, 0x4140);
        h[1] = prmt(w0, 0x64646464u, 0x4342);
        h[2] = prmt(w1, 0x64646464u, 0x4140);
        h[3] = prmt(w1, 0x64646464u, 0x4342);
      } else {        // 2 bytes (4 values each): bytes 2 ch, 2 ch + 1 of the 32 code bytes
        const uint4 cw = k.code[ch >> 3];
        const uint32_t wsel = ((ch >> 1) & 3) == 0 ? cw.x : (((ch >> 1) & 3) == 1 ? cw.y : (((ch >> 1) & 3) == 2 ? cw.z : cw.w));
        const uint32_t x = (wsel >> (16 * (ch & 1))) & 0xFFFFu;
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // values 2e, 2e+1 of the 8
          const uint32_t v0 = (x >> (4 * e)) & 3u, v1 = (x >> (4 * e + 2)) & 3u;
          h[e] = v0 | (v1 << 16) | 0x64006400u;
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) h[e] = hfma2_u(hsub2_u(h[e], H2_1024), s2, z2);
      *reinterpret_cast<uint4*>(stage + sw128_off(r, ch, KT * 128)) = make_uint4(h[0], h[1], h[2], h[3]);
    }
    return;
  }
  if (k.packed) {
    const uint32_t szw[4] = {k.sz.x, k.sz.y, k.sz.z, k.sz.w};
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {  // 16 code bytes = dims 32 q4 .. 32 q4 + 31 (group q4)
      const uint32_t s2 = prmt(szw[q4], szw[q4], 0x1010), z2 = prmt(szw[q4], szw[q4], 0x3232);
      const uint32_t wv[4] = {k.code[q4].x, k.code[q4].y, k.code[q4].z, k.code[q4].w};
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {  // word kk: dims 32 q4 + 8 kk .. + 7
        uint32_t h[4];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          // bytes 2e, 2e+1 at bits 0..7 and 16..23: low nibbles -> dims (4e, 4e+2),
          // high nibbles -> dims (4e+1, 4e+3)
          const uint32_t x = prmt(wv[kk], 0u, e ? 0x4342 : 0x4140);
          const uint32_t lo = hfma2_u(nib_lo(x), s2, z2);
          const uint32_t hi = hfma2_u(nib_hi(x), s2, z2);
          h[2 * e] = prmt(lo, hi, 0x5410);      // dims 4e, 4e+1
          h[2 * e + 1] = prmt(lo, hi, 0x7632);  // dims 4e+2, 4e+3
        }
        *reinterpret_cast<uint4*>(stage + sw128_off(r, 4 * q4 + kk, KT * 128)) = make_uint4(h[0], h[1], h[2], h[3]);
      }
    }
    return;
  }
#pragma unroll
  for (int ch = 0; ch < 16; ++ch) *reinterpret_cast<uint4*>(stage + sw128_off(r, ch, KT * 128)) = make_uint4(0u, 0u, 0u, 0u);
}

template <bool COL>
__global__ void __launch_bounds__(SEL_THREADS, 1) sel_pass(SelArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t kfull[2], kfree[2], tfull[4], tfree[4], drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const hq_cache& c = a.c;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int bh = b * c.Hkv + kvh;
  const int G = c.Hq / c.Hkv;
  const int Mp = a.Mp;
  const int NACC = Mp / 128;
  const SelGeo g = sel_geo(a, b);
  int32_t* const srow = state_row(c, b);
  const int M = G * g.nq;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Row normalisers from the decode steps: when every buffered query was
  // decoded after the last merge, its decode step saw exactly the keys this
  // reselection sees (same VL set, same packed range, the rest FP16), and the
  // log-sum-exp it stored is the one pass 0 would compute; pass 0 then only
  // clears its slice of the histogram.
  bool use_dec = false;
  if (!a.k_dense && c.qlse != nullptr && g.nq > 0 && g.qpos0 >= g.n_packed + c.W) {
    bool ok = true;
    for (int r = threadIdx.x; r < M; r += SEL_THREADS) {
      const int h = r / g.nq, p = g.qpos0 + r % g.nq;
      const float z = c.qlse[(static_cast<size_t>(b) * c.Hq + kvh * G + h) * HQ_QBUF + (p % HQ_QBUF)];
      ok = ok && isfinite(z);
    }
    use_dec = __syncthreads_and(ok) != 0;
  }
  if (!COL && use_dec) {
    uint32_t* gh = a.hist + static_cast<size_t>(bh) * HBINS;
    for (int e = (split * HBINS) / a.S + threadIdx.x; e < ((split + 1) * HBINS) / a.S; e += SEL_THREADS) gh[e] = 0u;
    return;
  }

  // this CTA's key tiles: pass 0 covers every visible key [0, T), pass 1 the
  // candidates [0, n)
  const int lim = COL ? g.n : g.T;
  const int ntl = (lim + KT - 1) / KT;
  const int k_lo = (split * ntl) / a.S, k_hi = ((split + 1) * ntl) / a.S;
  const int nt = M > 0 ? k_hi - k_lo : 0;
  // TMEM buffers: pass 0 holds NACC accumulators of 128 columns per tile,
  // pass 1 one accumulator of Mp columns
  const int NBUF = max(1, 4 / NACC);

  uint8_t* qs = sm;                          // 2 halves x [Mp][128 B]
  uint8_t* ks = sm + Mp * 256;               // 2 stages x KSTAGE
  float* aux = reinterpret_cast<float*>(ks + 2 * KSTAGE);
  int* qpos = reinterpret_cast<int*>(aux);   // [Mp] query positions
  float* lse = aux + Mp;                     // [Mp] pass 1: log-sum-exp (exp2 domain), +inf on padding rows
  float* xch = aux + 2 * Mp;                 // [2][Mp] pass 0 (m, l) of column half 1; pass 1 [KT] partial sums
  uint32_t* shist = reinterpret_cast<uint32_t*>(aux + 4 * Mp);  // [HBINS] pass 1: this CTA's score histogram

  if (threadIdx.x == 0) {
    mbar_init(&kfull[0], BLD_WARPS * 32);
    mbar_init(&kfull[1], BLD_WARPS * 32);
    mbar_init(&kfree[0], 1);
    mbar_init(&kfree[1], 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tfree[i], EPI_WARPS * 32);
    }
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  // queries: row r = h * nq + i (head kvh*G + h, position qpos0 + i); rows >= M are zero.
  // Asynchronous 16-byte copies, all in flight at once (waited for below).
  for (int e = threadIdx.x; e < Mp * (D / 8); e += SEL_THREADS) {
    const int r = e / (D / 8), ch = e % (D / 8);
    uint8_t* dst = qs + sw128_off(r, ch, Mp * 128);
    if (r < M) {
      const int h = r / g.nq, i = r % g.nq;
      const uint4* src;
      if (a.k_dense) {
        src = reinterpret_cast<const uint4*>(a.q_ext + ((static_cast<size_t>(b) * c.Hq + kvh * G + h) * g.nq + i) * D) + ch;
      } else {
        const int p = g.qpos0 + i;
        src = reinterpret_cast<const uint4*>(c.qbuf + ((static_cast<size_t>(b) * c.Hq + kvh * G + h) * HQ_QBUF + (p % HQ_QBUF)) * D) + ch;
      }
      cp_async16(dst, src);
    } else {
      *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  for (int r = threadIdx.x; r < Mp; r += SEL_THREADS) qpos[r] = r < M ? g.qpos0 + r % max(g.nq, 1) : -1;
  if (!COL) {
    // the head's score histogram is rebuilt by pass 1: each split clears a slice
    uint32_t* gh = a.hist + static_cast<size_t>(bh) * HBINS;
    for (int e = (split * HBINS) / a.S + threadIdx.x; e < ((split + 1) * HBINS) / a.S; e += SEL_THREADS) gh[e] = 0u;
  } else {
    for (int e = threadIdx.x; e < HBINS; e += SEL_THREADS) shist[e] = 0u;
  }
  if (COL) {
    // per-row log-sum-exp: stored by the decode steps, or over the pass-0 partials of every split
    for (int r = threadIdx.x; r < Mp; r += SEL_THREADS) {
      float z = INFINITY;
      if (r < M && use_dec) {
        const int h = r / g.nq, p = g.qpos0 + r % g.nq;
        z = c.qlse[(static_cast<size_t>(b) * c.Hq + kvh * G + h) * HQ_QBUF + (p % HQ_QBUF)];
      } else if (r < M) {
        const float* lp = a.lse_part + (static_cast<size_t>(bh) * MAX_SPLITS) * Mp * 2 + 2 * r;
        float mm = -INFINITY, ll = 0.f;
#pragma unroll 8
        for (int sp = 0; sp < a.S; ++sp) {
          const float2 ml = __ldcg(reinterpret_cast<const float2*>(lp + static_cast<size_t>(sp) * Mp * 2));
          const float mn = fmaxf(mm, ml.x);
          if (mn != -INFINITY) {
            ll = ll * ex2(mm - mn) + ml.y * ex2(ml.x - mn);
            mm = mn;
          }
        }
        z = mm + log2f(ll);
      }
      lse[r] = z;
    }
  }
  cp_async_wait_all();  // this thread's query copies
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t sbase = smem_u32(sm);

  if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t q_s = sbase, k_s = sbase + Mp * 256;
      bool ok = true;
      for (int t = 0; t < nt && ok; ++t) {
        const int s = t & 1, buf = t % NBUF;
        ok = sel_wait(&kfull[s], (t >> 1) & 1, srow, &abort_flag);
        if (ok && t >= NBUF) ok = sel_wait(&tfree[buf], ((t / NBUF) - 1) & 1, srow, &abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kst = k_s + s * KSTAGE;
        if (!COL) {
          constexpr uint32_t IDESC = idesc_make(0, 0, 0, 128, KT);
          for (int acc = 0; acc < NACC; ++acc) {
            const uint32_t d = tmem + (buf * NACC + acc) * 128;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t ao = (kk >> 2) * (Mp * 128) + acc * 16384 + 32 * (kk & 3);
              const uint32_t bo = (kk >> 2) * (KT * 128) + 32 * (kk & 3);
              umma_f16(d, sdesc_sw128(q_s + ao, 16, 1024), sdesc_sw128(kst + bo, 16, 1024), IDESC, kk > 0);
            }
          }
        } else {
          for (int nh = 0; nh * 256 < Mp; ++nh) {
            const int N = min(256, Mp - 256 * nh);
            const uint32_t idesc = idesc_make(0, 0, 0, 128, N);
            const uint32_t d = tmem + buf * Mp + 256 * nh;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t ao = (kk >> 2) * (KT * 128) + 32 * (kk & 3);
              const uint32_t bo = (kk >> 2) * (Mp * 128) + nh * 256 * 128 + 32 * (kk & 3);
              umma_f16(d, sdesc_sw128(kst + ao, 16, 1024), sdesc_sw128(q_s + bo, 16, 1024), idesc, kk > 0);
            }
          }
        }
        umma_commit(&tfull[buf]);
        umma_commit(&kfree[s]);
      }
      // every MMA issued completes before TMEM is released
      umma_commit(&drain);
      int dummy = 0;
      sel_wait(&drain, 0, srow, &dummy);
    }
    __syncwarp();
  } else if (warp >= EPI_WARPS) {
    // ------------------------------------------------------------ key builders
    // one key row per thread; the next tile's row is fetched before this one
    // is converted, so its load latency hides behind the conversion
    const int r = threadIdx.x - EPI_WARPS * 32;
    KeyRow cur = fetch_key_row(a, g, bh, k_lo * KT + r);
    for (int t = 0; t < nt; ++t) {
      const int s = t & 1;
      const KeyRow nxt = t + 1 < nt ? fetch_key_row(a, g, bh, (k_lo + t + 1) * KT + r) : cur;
      if (t >= 2 && !__all_sync(0xffffffffu, sel_wait(&kfree[s], ((t >> 1) - 1) & 1, srow, &abort_flag))) break;
      store_key_row(a, bh, cur, ks + s * KSTAGE, r);
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(&kfull[s]);
      cur = nxt;
      // the next tile's loads are back by now: warm L2 with its vertical lines' rows
      if (t + 1 < nt && cur.packed) {
        const uint4* vsrc = key_row_src(a, bh, cur);
        if (vsrc) prefetch_l2(vsrc, D * 2);
      }
    }
  } else if (COL && M == 0) {
    // no buffered queries: every candidate's column mass is zero
    for (int j = k_lo * KT + threadIdx.x; j < min(k_hi * KT, g.n); j += EPI_WARPS * 32)
      a.scores[static_cast<size_t>(bh) * c.cap + j] = 0.f;
    if (threadIdx.x == 0 && min(k_hi * KT, g.n) > k_lo * KT)
      atomicAdd(a.hist + static_cast<size_t>(bh) * HBINS, static_cast<unsigned>(min(k_hi * KT, g.n) - k_lo * KT));
  } else {
    // ------------------------------------------------------------ epilogue
    const int qd = warp & 3, hc = warp >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
    if (!COL) {
      // thread: query row acc * 128 + 32 qd + lane of every accumulator, key
      // columns [64 hc, 64 hc + 64) of each tile
      float m_run[4], l_run[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { m_run[i] = -INFINITY; l_run[i] = 0.f; }
      for (int t = 0; t < nt; ++t) {
        const int buf = t % NBUF;
        if (!__all_sync(0xffffffffu, sel_wait(&tfull[buf], (t / NBUF) & 1, srow, &abort_flag))) break;
        tc_fence_after();
        const int j0 = (k_lo + t) * KT + 64 * hc;
#pragma unroll
        for (int acc = 0; acc < 4; ++acc) {
          if (acc >= NACC) break;
          const int row = acc * 128 + qd * 32 + lane;
          const int p = qpos[row];
          // keys j0 + c visible to this row: c <= min(p, T - 1) - j0
          const int cmax = min(p, g.T - 1) - j0;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t u[32];
            tmem_ld32(tmem + lane_base + (buf * NACC + acc) * 128 + 64 * hc + 32 * h, u);
            tmem_wait_ld();
            float mx = -INFINITY;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float x = (32 * h + e <= cmax) ? __uint_as_float(u[e]) * a.qscale : -INFINITY;
              u[e] = __float_as_uint(x);
              mx = fmaxf(mx, x);
            }
            // lazy running max: move it only when the chunk max exceeds it by > 2^8
            if (mx > m_run[acc] + 8.0f) {
              l_run[acc] *= ex2(m_run[acc] - mx);
              m_run[acc] = mx;
            }
            const float ref = m_run[acc] == -INFINITY ? 0.f : m_run[acc];
            float l0 = 0.f, l1 = 0.f;
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              l0 += ex2(__uint_as_float(u[e]) - ref);
              l1 += ex2(__uint_as_float(u[e + 1]) - ref);
            }
            l_run[acc] += l0 + l1;
          }
        }
        tc_fence_before();
        mbar_arrive(&tfree[buf]);
      }
      // merge the two column halves, then the partial (m, l) of each row
      if (hc == 1) {
#pragma unroll
        for (int acc = 0; acc < 4; ++acc) {
          if (acc >= NACC) break;
          const int row = acc * 128 + qd * 32 + lane;
          xch[2 * row] = m_run[acc];
          xch[2 * row + 1] = l_run[acc];
        }
      }
      asm volatile("bar.sync 1, %0;" ::"r"(EPI_WARPS * 32) : "memory");
      if (hc == 0) {
        float* lp = a.lse_part + ((static_cast<size_t>(bh) * MAX_SPLITS + split) * Mp) * 2;
#pragma unroll
        for (int acc = 0; acc < 4; ++acc) {
          if (acc >= NACC) break;
          const int row = acc * 128 + qd * 32 + lane;
          const float m1 = xch[2 * row], l1 = xch[2 * row + 1];
          const float mm = fmaxf(m_run[acc], m1);
          float ll = 0.f;
          if (mm != -INFINITY) ll = l_run[acc] * ex2(m_run[acc] - mm) + l1 * ex2(m1 - mm);
          lp[2 * row] = mm;
          lp[2 * row + 1] = ll;
        }
      }
    } else {
      // thread: key qd * 32 + lane of each tile, query columns [hc Mp/2, (hc+1) Mp/2)
      const int half = Mp / 2;
      for (int t = 0; t < nt; ++t) {
        const int buf = t % NBUF;
        if (!__all_sync(0xffffffffu, sel_wait(&tfull[buf], (t / NBUF) & 1, srow, &abort_flag))) break;
        tc_fence_after();
        const int j = (k_lo + t) * KT + qd * 32 + lane;
        // queries that may not see key j: positions < j (only near the end)
        const bool all_see = j <= g.qpos0;
        float sum = 0.f;
        for (int c0 = hc * half; c0 < (hc + 1) * half; c0 += 32) {
          uint32_t u[32];
          tmem_ld32(tmem + lane_base + buf * Mp + c0, u);
          tmem_wait_ld();
          float s0 = 0.f, s1 = 0.f;
          const float4* lz = reinterpret_cast<const float4*>(lse + c0);
          if (all_see) {
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
              const float4 z = lz[e4];
              s0 += ex2(fmaf(__uint_as_float(u[4 * e4]), a.qscale, -z.x));
              s1 += ex2(fmaf(__uint_as_float(u[4 * e4 + 1]), a.qscale, -z.y));
              s0 += ex2(fmaf(__uint_as_float(u[4 * e4 + 2]), a.qscale, -z.z));
              s1 += ex2(fmaf(__uint_as_float(u[4 * e4 + 3]), a.qscale, -z.w));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float v = ex2(fmaf(__uint_as_float(u[e]), a.qscale, -lse[c0 + e]));
              s0 += qpos[c0 + e] >= j ? v : 0.f;
            }
          }
          sum += s0 + s1;
        }
        tc_fence_before();
        mbar_arrive(&tfree[buf]);
        // the two column halves of key j: half 1 hands its sum over, half 0 writes
        if (hc == 1) xch[qd * 32 + lane] = sum;
        asm volatile("bar.sync 1, %0;" ::"r"(EPI_WARPS * 32) : "memory");
        if (hc == 0 && j < g.n) {
          float sc_j = sum + xch[qd * 32 + lane];
          if (c.score_acc) {  // running scores: decode mode adds to the stored sum, init mode starts it
            float* acc = c.score_acc + static_cast<size_t>(bh) * c.cap + j;
            if (!a.k_dense) sc_j += *acc;
            *acc = sc_j;
          }
          a.scores[static_cast<size_t>(bh) * c.cap + j] = sc_j;
          atomicAdd(shist + (__float_as_uint(sc_j) >> 20), 1u);
        }
        asm volatile("bar.sync 1, %0;" ::"r"(EPI_WARPS * 32) : "memory");
      }
      // this CTA's histogram into the head's
      uint32_t* gh = a.hist + static_cast<size_t>(bh) * HBINS;
      for (int e = threadIdx.x; e < HBINS; e += EPI_WARPS * 32)
        if (shist[e]) atomicAdd(gh + e, shist[e]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

constexpr int TK_THREADS = 1024;
constexpr int TK_SMEM_MAX = 47104;  // scores held in shared memory up to this many candidates (with the static arrays, <= 227 KB)
constexpr int TK_CAND_MAX = 8192;   // values of the threshold's histogram bin held in shared memory

// Exact top-k of the column-mass scores of one (b, kv head).  Scores are >= 0,
// so their fp32 bit patterns order like the values.  (1) The histogram of bits
// 30..20 that the column-mass pass built gives the bin holding the k-th
// largest value and how many values lie above it.  (2) The values of that bin
// are gathered into shared memory.  (3) Its low 20 bits are found by two radix
// passes of 10 bits (a 1024-bin histogram of the candidates, then the sub-bin
// holding the needed rank).  (4) An ordered compaction, one contiguous range
// of positions per warp, writes the chosen positions ascending, ties at the
// threshold to the lowest positions.  A bin too large for shared memory is
// searched in global memory.
__global__ void __launch_bounds__(TK_THREADS) topk_kernel(SelArgs a, int smem_scores) {
  const hq_cache& c = a.c;
  const int bh = blockIdx.x;
  const int b = bh / c.Hkv;
  int32_t* const srow = state_row(c, b);
  const SelGeo g = sel_geo(a, b);
  const int n = g.n;
  int k = 0;
  if (n > 0 && c.rho_bp > 0) {
    const long long kk = (static_cast<long long>(n) * c.rho_bp + 9999) / 10000;
    k = static_cast<int>(min(static_cast<long long>(n), kk));
  }
  if (k > c.vl_cap) {
    if (bh % c.Hkv == 0 && threadIdx.x == 0) set_err(srow, HQ_DEVERR_VL_CAPACITY);
    k = c.vl_cap;
  }
  if (bh % c.Hkv == 0 && threadIdx.x == 0) srow[HQ_STATE_KSEL] = k;
  if (k == 0) return;
  extern __shared__ uint32_t tk_smem[];  // [TK_CAND_MAX] bin values, then [smem_scores] scores
  __shared__ unsigned int s_bin, s_above, s_cnt;
  __shared__ unsigned int wsum[TK_THREADS / 32];
  __shared__ unsigned int tk_hist[TK_THREADS];   // radix sub-bins of the threshold bin
  const uint32_t* gsc = reinterpret_cast<const uint32_t*>(a.scores + static_cast<size_t>(bh) * c.cap);
  uint32_t* cand = tk_smem;
  // the scores are staged in shared memory (all loads in flight at once) when they fit
  const bool staged = n <= smem_scores;
  uint32_t* ssc = tk_smem + TK_CAND_MAX;
  if (staged) {
#pragma unroll 8
    for (int j = threadIdx.x; j < n; j += TK_THREADS) ssc[j] = __ldcg(gsc + j);
  }
  const uint32_t* sc = staged ? ssc : gsc;
  const uint32_t* hh = a.hist + static_cast<size_t>(bh) * HBINS;
  int32_t* out = c.vl_sel + static_cast<size_t>(bh) * c.vl_cap;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // (1) thread i owns bins 2047 - 2i (higher) and 2046 - 2i; an inclusive scan
  // over threads gives the suffix sums S_d = #values in bins >= d
  {
    const int d1 = HBINS - 1 - 2 * threadIdx.x, d0 = d1 - 1;
    const unsigned int h1 = __ldcg(hh + d1), h0 = __ldcg(hh + d0);
    unsigned int x = h1 + h0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    if (threadIdx.x == 0) {
      s_cnt = 0u;
      s_bin = 0u;  // only if the histogram disagreed with the scores (never expected)
      s_above = 0u;
    }
    __syncthreads();
    for (int w = 0; w < warp; ++w) x += wsum[w];
    const unsigned int S0 = x, S1 = x - h0, Sabove = x - h0 - h1;  // S_{d0}, S_{d1}, S_{d1+1}
    const unsigned int kk = static_cast<unsigned int>(k);
    if (S1 >= kk && Sabove < kk) {
      s_bin = d1;
      s_above = Sabove;
    } else if (S0 >= kk && S1 < kk) {
      s_bin = d0;
      s_above = S1;
    }
    __syncthreads();
  }
  const uint32_t bin = s_bin;
  const unsigned int need = static_cast<unsigned int>(k) - min(s_above, static_cast<unsigned int>(k) - 1u);  // >= 1
  const unsigned int nbin = __ldcg(hh + bin);
  const bool in_smem = nbin <= static_cast<unsigned int>(TK_CAND_MAX);
  // (2) the bin's values
  if (in_smem) {
    for (int j0 = 0; j0 < n; j0 += TK_THREADS) {
      const int j = j0 + threadIdx.x;
      const uint32_t v = j < n ? sc[j] : 0u;
      const bool hit = j < n && (v >> 20) == bin;
      const unsigned int m = __ballot_sync(0xffffffffu, hit);
      unsigned int base = 0u;
      if (lane == 0 && m) base = atomicAdd(&s_cnt, static_cast<unsigned>(__popc(m)));
      base = __shfl_sync(0xffffffffu, base, 0);
      const unsigned int slot = base + __popc(m & ((1u << lane) - 1u));
      if (hit && slot < nbin) cand[slot] = v;  // nbin <= TK_CAND_MAX: the list never overflows
    }
  }
  __syncthreads();
  const int ncand = in_smem ? static_cast<int>(min(s_cnt, nbin)) : n;
  // (3) the low 20 bits of the k-th largest, by two radix passes of 10 bits over
  // the bin's values: a 1024-bin histogram of bits 19..10, the sub-bin holding
  // the needed rank, then a histogram of bits 9..0 inside that sub-bin
  unsigned int* h10 = tk_hist;
  uint32_t prefix = bin << 20;   // bits fixed so far
  uint32_t pmask = 0xFFF00000u;  // which bits are fixed
  unsigned int above = s_above;  // values above everything that matches the prefix
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = pass == 0 ? 10 : 0;
    h10[threadIdx.x] = 0u;
    __syncthreads();
    for (int e = threadIdx.x; e < ncand; e += TK_THREADS) {
      const uint32_t v = in_smem ? cand[e] : sc[e];
      if ((v & pmask) == prefix) atomicAdd(&h10[(v >> shift) & 1023u], 1u);
    }
    __syncthreads();
    // suffix sums over the 1024 sub-bins, highest first: thread i owns sub-bin 1023 - i
    const unsigned int hv = h10[TK_THREADS - 1 - threadIdx.x];
    unsigned int x = hv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    for (int w = 0; w < warp; ++w) x += wsum[w];
    // x = values in sub-bins >= this one (within the prefix); the needed rank is k - above
    const unsigned int needp = static_cast<unsigned int>(k) - above;
    if (x >= needp && x - hv < needp) {
      s_bin = TK_THREADS - 1 - threadIdx.x;
      s_above = above + (x - hv);
      s_cnt = hv;
    }
    __syncthreads();
    prefix |= s_bin << shift;
    pmask |= 1023u << shift;
    above = s_above;
    __syncthreads();
  }
  const uint32_t thr = prefix;
  // take_eq of the values equal to thr (the lowest positions), all values above it
  const unsigned int take_eq = static_cast<unsigned int>(k) - above;
  // (4) ordered compaction: warp w owns positions [w P, (w + 1) P); a first
  // sweep counts the values above and equal to thr per warp, a block scan gives
  // each warp its output offsets, a second sweep writes positions in order
  // (ballots inside the warp, 32 consecutive positions per round)
  const int P = ((n + TK_THREADS / 32 - 1) / (TK_THREADS / 32) + 31) / 32 * 32;
  const int j_lo = warp * P, j_hi = min(n, j_lo + P);
  unsigned int cg = 0u, ce = 0u;
  for (int j0 = j_lo; j0 < j_hi; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t v = j < j_hi ? sc[j] : 0u;
    cg += __popc(__ballot_sync(0xffffffffu, j < j_hi && v > thr));
    ce += __popc(__ballot_sync(0xffffffffu, j < j_hi && v == thr));
  }
  __shared__ unsigned int rg[TK_THREADS / 32], re[TK_THREADS / 32];
  if (lane == 0) {
    rg[warp] = cg;
    re[warp] = ce;
  }
  __syncthreads();
  unsigned int xg = 0u, xe = 0u;
  for (int w = 0; w < warp; ++w) {
    xg += rg[w];
    xe += re[w];
  }
  const unsigned int lt_mask = (1u << lane) - 1u;
  for (int j0 = j_lo; j0 < j_hi; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t v = j < j_hi ? sc[j] : 0u;
    const bool gt = j < j_hi && v > thr, eq = j < j_hi && v == thr;
    const unsigned int bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
    const unsigned int mg = xg + __popc(bg & lt_mask), me = xe + __popc(be & lt_mask);
    if (gt) out[mg + min(me, take_eq)] = j;
    else if (eq && me < take_eq) out[mg + me] = j;
    xg += __popc(bg);
    xe += __popc(be);
  }
}


// The same top-k spread over a cluster of TKC_CS CTAs per (b, kv head): CTA r
// owns positions [r P, (r + 1) P).  Each CTA takes the threshold bin from the
// global histogram, gathers its range's values of that bin, and builds a local
// histogram of each radix pass; the cluster sums the local histograms through
// distributed shared memory, so every CTA finds the same sub-bin.  The ordered
// compaction offsets each CTA by the counts of the lower-ranked CTAs (read the
// same way).  Same result as topk_kernel, bit for bit.
constexpr int TKC_CS = 8;                 // CTAs per (b, kv head): one portable cluster
constexpr int TKC_THREADS = 512;
constexpr int TKC_PMAX = 24576;           // positions per CTA held in shared memory (scores and bin values)

__device__ __forceinline__ unsigned int tkc_block_scan(unsigned int x, unsigned int* wsum, int lane, int warp) {
  // inclusive scan over the block's threads in thread order
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  for (int w = 0; w < warp; ++w) x += wsum[w];
  return x;
}

__global__ void __cluster_dims__(TKC_CS, 1, 1) __launch_bounds__(TKC_THREADS) topk_cluster_kernel(SelArgs a) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const hq_cache& c = a.c;
  const int rank = static_cast<int>(cl.block_rank());
  const int bh = blockIdx.x / TKC_CS;
  const int b = bh / c.Hkv;
  int32_t* const srow = state_row(c, b);
  const SelGeo g = sel_geo(a, b);
  const int n = g.n;
  int k = 0;
  if (n > 0 && c.rho_bp > 0) {
    const long long kk = (static_cast<long long>(n) * c.rho_bp + 9999) / 10000;
    k = static_cast<int>(min(static_cast<long long>(n), kk));
  }
  if (k > c.vl_cap) {
    if (rank == 0 && bh % c.Hkv == 0 && threadIdx.x == 0) set_err(srow, HQ_DEVERR_VL_CAPACITY);
    k = c.vl_cap;
  }
  if (rank == 0 && bh % c.Hkv == 0 && threadIdx.x == 0) srow[HQ_STATE_KSEL] = k;
  if (k == 0) return;  // the same for every CTA of the cluster: no shared-memory exchange follows
  extern __shared__ uint32_t tkc_smem[];  // [P] scores of the range, then [P] values of the threshold bin
  __shared__ unsigned int h10[2][1024];    // local histograms of the two radix passes
  __shared__ unsigned int wsum[TKC_THREADS / 32], rg[TKC_THREADS / 32], re[TKC_THREADS / 32];
  __shared__ unsigned int s_bin, s_above, s_cnt, s_tot[2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int P = ((n + TKC_CS - 1) / TKC_CS + 31) / 32 * 32;
  const int lo = min(n, rank * P), hi = min(n, lo + P), m = hi - lo;
  uint32_t* sc = tkc_smem;
  uint32_t* cand = tkc_smem + P;
  const uint32_t* gsc = reinterpret_cast<const uint32_t*>(a.scores + static_cast<size_t>(bh) * c.cap);
#pragma unroll 4
  for (int j = threadIdx.x; j < m; j += TKC_THREADS) sc[j] = __ldcg(gsc + lo + j);
  const uint32_t* hh = a.hist + static_cast<size_t>(bh) * HBINS;
  int32_t* out = c.vl_sel + static_cast<size_t>(bh) * c.vl_cap;
  for (int e = threadIdx.x; e < 2 * 1024; e += TKC_THREADS) (&h10[0][0])[e] = 0u;  // before the barriers below

  // (1) the threshold bin: thread i owns bins 2047 - 4i .. 2044 - 4i (descending)
  {
    const int d_hi = HBINS - 1 - 4 * static_cast<int>(threadIdx.x);
    unsigned int h[4], x = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      h[j] = __ldcg(hh + d_hi - j);
      x += h[j];
    }
    if (threadIdx.x == 0) {
      s_bin = 0u;  // only if the histogram disagreed with the scores (never expected)
      s_above = 0u;
      s_cnt = 0u;
    }
    const unsigned int X = tkc_block_scan(x, wsum, lane, warp);
    unsigned int above = X - x;  // values in bins > d_hi
    const unsigned int kk = static_cast<unsigned int>(k);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (above < kk && above + h[j] >= kk) {
        s_bin = static_cast<unsigned int>(d_hi - j);
        s_above = above;
      }
      above += h[j];
    }
    __syncthreads();
  }
  const uint32_t bin = s_bin;
  // (2) this range's values of the threshold bin
  for (int j0 = 0; j0 < m; j0 += TKC_THREADS) {
    const int j = j0 + threadIdx.x;
    const uint32_t v = j < m ? sc[j] : 0u;
    const bool hit = j < m && (v >> 20) == bin;
    const unsigned int msk = __ballot_sync(0xffffffffu, hit);
    unsigned int base = 0u;
    if (lane == 0 && msk) base = atomicAdd(&s_cnt, static_cast<unsigned>(__popc(msk)));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (hit) cand[base + __popc(msk & ((1u << lane) - 1u))] = v;  // at most m <= P values
  }
  __syncthreads();
  const int ncand = static_cast<int>(s_cnt);
  // (3) the low 20 bits of the k-th largest: two radix passes of 10 bits, the
  // cluster's histograms summed from every CTA's shared memory (one histogram
  // per pass, so no CTA has to wait for the others' reads before the next)
  uint32_t prefix = bin << 20, pmask = 0xFFF00000u;
  unsigned int above = s_above;
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = pass == 0 ? 10 : 0;
    for (int e = threadIdx.x; e < ncand; e += TKC_THREADS) {
      const uint32_t v = cand[e];
      if ((v & pmask) == prefix) atomicAdd(&h10[pass][(v >> shift) & 1023u], 1u);
    }
    cl.sync();  // every CTA's histogram complete
    // thread i owns sub-bins 1023 - 2i and 1022 - 2i (descending)
    const int d1 = 1023 - 2 * static_cast<int>(threadIdx.x), d0 = d1 - 1;
    unsigned int g1 = 0u, g0 = 0u;
#pragma unroll
    for (int r = 0; r < TKC_CS; ++r) {
      const unsigned int* rh = cl.map_shared_rank(&h10[pass][0], r);
      g1 += rh[d1];
      g0 += rh[d0];
    }
    const unsigned int X = tkc_block_scan(g1 + g0, wsum, lane, warp);
    const unsigned int up = X - g1 - g0;  // values (within the prefix) in sub-bins above d1
    const unsigned int needp = static_cast<unsigned int>(k) - above;
    if (up < needp && up + g1 >= needp) {
      s_bin = static_cast<unsigned int>(d1);
      s_above = above + up;
    } else if (up + g1 < needp && up + g1 + g0 >= needp) {
      s_bin = static_cast<unsigned int>(d0);
      s_above = above + up + g1;
    }
    __syncthreads();
    prefix |= s_bin << shift;
    pmask |= 1023u << shift;
    above = s_above;
    __syncthreads();
  }
  const uint32_t thr = prefix;
  const unsigned int take_eq = static_cast<unsigned int>(k) - above;
  // (4) ordered compaction: warp w owns the range's positions [w Pw, (w + 1) Pw);
  // counts per warp, per CTA, then the lower-ranked CTAs' totals give the offsets
  const int Pw = ((m + TKC_THREADS / 32 - 1) / (TKC_THREADS / 32) + 31) / 32 * 32;
  const int j_lo = min(m, warp * Pw), j_hi = min(m, j_lo + Pw);
  unsigned int cg_ = 0u, ce = 0u;
  for (int j0 = j_lo; j0 < j_hi; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t v = j < j_hi ? sc[j] : 0u;
    cg_ += __popc(__ballot_sync(0xffffffffu, j < j_hi && v > thr));
    ce += __popc(__ballot_sync(0xffffffffu, j < j_hi && v == thr));
  }
  if (lane == 0) {
    rg[warp] = cg_;
    re[warp] = ce;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned int tg = 0u, te = 0u;
    for (int w = 0; w < TKC_THREADS / 32; ++w) {
      tg += rg[w];
      te += re[w];
    }
    s_tot[0] = tg;
    s_tot[1] = te;
  }
  cl.sync();  // every CTA's totals visible
  unsigned int xg = 0u, xe = 0u;
  for (int r = 0; r < rank; ++r) {
    const unsigned int* rt = cl.map_shared_rank(s_tot, r);
    xg += rt[0];
    xe += rt[1];
  }
  // done reading the other CTAs' shared memory: arrive now, wait before leaving
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  for (int w = 0; w < warp; ++w) {
    xg += rg[w];
    xe += re[w];
  }
  const unsigned int lt_mask = (1u << lane) - 1u;
  for (int j0 = j_lo; j0 < j_hi; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t v = j < j_hi ? sc[j] : 0u;
    const bool gt = j < j_hi && v > thr, eq = j < j_hi && v == thr;
    const unsigned int bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
    const unsigned int mg = xg + __popc(bg & lt_mask), me = xe + __popc(be & lt_mask);
    // (the bounds hold whenever the histogram agrees with the scores, as it does by construction)
    const unsigned int kk = static_cast<unsigned int>(k);
    if (gt && mg + min(me, take_eq) < kk) out[mg + min(me, take_eq)] = lo + j;
    else if (eq && me < take_eq && mg + me < kk) out[mg + me] = lo + j;
    xg += __popc(bg);
    xe += __popc(be);
  }
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");  // no CTA leaves while another may still read its shared memory
}

int sel_mp(const hq_cache& c) { return (((c.Hq / c.Hkv) * HQ_QBUF + 127) / 128) * 128; }

size_t sel_smem_bytes(int Mp) {
  return 1024 + static_cast<size_t>(Mp) * 256 + 2 * KSTAGE + 4 * static_cast<size_t>(Mp) * 4 + HBINS * 4;
}

}  // namespace

size_t select_workspace(const hq_cache& c, bool need_scores) {
  const int Mp = sel_mp(c);
  size_t bytes = static_cast<size_t>(c.B) * c.Hkv * MAX_SPLITS * Mp * 2 * 4;  // (m, l) partials
  bytes += static_cast<size_t>(c.B) * c.Hkv * HBINS * 4;                       // score histograms
  if (need_scores) bytes += static_cast<size_t>(c.B) * c.Hkv * c.cap * 4;
  return (bytes + 255) & ~static_cast<size_t>(255);
}

hq_status launch_select(const hq_cache& c, const uint16_t* kd, int L, const uint16_t* qe, int nq, float* scores_out,
                        void* ws, cudaStream_t st) {
  SelArgs a;
  a.c = c;
  a.k_dense = kd;
  a.q_ext = qe;
  a.L = L;
  a.nq_init = nq;
  a.Mp = sel_mp(c);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int units = c.B * c.Hkv;
  int S = sms / units;
  const int keys_cap = kd ? L : c.cap;
  S = min(S, (keys_cap + KT - 1) / KT);
  S = max(1, min(S, MAX_SPLITS));
  a.S = S;
  char* w = static_cast<char*>(ws);
  a.lse_part = reinterpret_cast<float*>(w);
  w += static_cast<size_t>(c.B) * c.Hkv * MAX_SPLITS * a.Mp * 2 * 4;
  a.hist = reinterpret_cast<uint32_t*>(w);
  w += static_cast<size_t>(c.B) * c.Hkv * HBINS * 4;
  a.scores = scores_out ? scores_out : reinterpret_cast<float*>(w);
  a.qscale = (1.0f / sqrtf(static_cast<float>(D))) * LOG2E;
  const size_t smem = sel_smem_bytes(a.Mp);
  static DeviceOnce attrs;
  const cudaError_t ea = attrs.run(dev, [] {
    const int smem_max = static_cast<int>(sel_smem_bytes(((HQ_MAX_GQA * HQ_QBUF + 127) / 128) * 128));
    cudaError_t e = cudaFuncSetAttribute(sel_pass<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(sel_pass<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (TK_CAND_MAX + TK_SMEM_MAX) * 4);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * TKC_PMAX * 4);
    return e;
  });
  if (ea != cudaSuccess) return cuda_fail(ea, "select setup");
  if (kd != nullptr && c.score_acc != nullptr &&
      cudaMemsetAsync(c.score_acc, 0, static_cast<size_t>(c.B) * c.Hkv * c.cap * sizeof(float), st) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "select setup");
  dim3 grid(S, c.Hkv, c.B);
  sel_pass<false><<<grid, SEL_THREADS, smem, st>>>(a);
  sel_pass<true><<<grid, SEL_THREADS, smem, st>>>(a);
  // top-k: a cluster of TKC_CS CTAs per (b, kv head) when a CTA's range of
  // the candidates fits its shared memory, else one CTA per (b, kv head)
  const int n_max = max(keys_cap - c.W, 0);
  const int P_max = ((n_max + TKC_CS - 1) / TKC_CS + 31) / 32 * 32;
  if (P_max <= TKC_PMAX) {
    topk_cluster_kernel<<<c.B * c.Hkv * TKC_CS, TKC_THREADS, static_cast<size_t>(2 * max(P_max, 32)) * 4, st>>>(a);
  } else {
    // shared memory: the bin's values and, when they fit, the scores themselves
    const int smem_scores = min(n_max, TK_SMEM_MAX);
    topk_kernel<<<c.B * c.Hkv, TK_THREADS, static_cast<size_t>(TK_CAND_MAX + smem_scores) * 4, st>>>(a, smem_scores);
  }
  return cuda_status(cudaGetLastError(), "select launch");
}

}  // namespace hq
