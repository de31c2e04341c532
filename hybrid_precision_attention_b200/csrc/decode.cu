// decode.cu — one decode step of attention over the hybrid K4V4 / FP16 cache.
//
// HyQuant digest (agihunt.info), prefill/decode paragraph, and the repository
// README, Overview item 3: the decode cache stores most positions K4V4 and the
// vertical-line and recent positions FP16, and dequantisation is fused into the
// attention scan (online softmax over quantised blocks) so no FP16 cache is
// materialised.  The pages' kernel is Triton for SM80+; this is a B200 design.
//
// Design (bandwidth-bound: ~160 B of K4V4 per token and kv head):
//   * work: every (b, kv head) is a unit whose tile list holds its packed
//     tiles (one sub-page of 64 positions, or 32 when K and V take more than 8
//     bits together: K codes, V codes, their scale/zero words, then the page's
//     VL bitmap), its FP16 tiles (16 rows of the VL store, 16 slots of the
//     FP16 ring, which is a multiple of 16 long, so a tile is one contiguous
//     copy) and a last tile with the new token read straight from its input
//     pointer; a CTA runs its packed tiles first, then its FP16 ones;
//   * grid: persistent, one CTA per SM, each sequence with its own state row.
//     Few units (4 CTAs or more each): every unit gets its own CTAs in
//     proportion to its tiles, each an even share of the unit's packed and
//     FP16 tiles (the last 12 CTAs, which the scheduler starts last, stay
//     idle).  Many units (stream-K): the units' tile lists are concatenated
//     and cut into equal contiguous ranges, one per CTA, so every SM streams
//     the same number of tiles whatever the batch size or the sequences'
//     lengths; a range may cover parts of several units, one segment per
//     unit, and a small phantom weight per unit bounds the segments of a
//     range.  The plan is made before the dependency wait and kept when the
//     lengths it used did not change;
//   * a producer warp streams tiles into a 2 NC-stage shared-memory ring with
//     large 1-D bulk async copies (cp.async.bulk, mbarrier completion, no
//     multicast): 1 copy per packed tile, 2 per FP16 tile;
//   * NC consumer warps take tiles round-robin, each owning 2 of the 2 NC
//     stages (tile i -> stage i % 2NC -> warp i % NC), so every stage has a
//     single consumer and a waiter is never a full barrier phase behind.
//     Codes become fp16 in registers (exponent-bias tricks for 2-, 4- and
//     8-bit codes + one fma with the group's scale/zero; the kernel is
//     instantiated per code width), and both products run on tensor cores with
//     mma.m16n8k16 (f32 accumulate):
//       S^T[keys x 8 queries] = K^ (16 keys x 16 dims) . Q^T
//       O^T[dims x 8 queries] += V^T (16 dims x 16 keys) . P^T
//     P^T comes from the S^T accumulators by an 8x8 movmatrix transpose.  Dims
//     and keys are permuted inside each MMA so that every thread dequantises one
//     whole group from contiguous nibbles and the packed-tile shared-memory
//     reads are free of bank conflicts;
//   * per-warp online softmax in the exp2 domain.  At the end of a segment
//     every consumer warp leaves its state in the stage of its last tile (held
//     back from the producer until the merge is done), the consumers merge the
//     warp states into the segment's partial (m, l, O) in the workspace, and
//     the last CTA to finish a unit merges that unit's partials with a
//     log-sum-exp (an acquire-release ticket, no waiting), writes each query's
//     log-sum-exp for the next reselection, appends the unit's new token to
//     the ring and its queries to the query buffer (every CTA of the unit is
//     done reading by then); the last CTA to take its grid ticket (taken with
//     the unit ticket, once it has read every length it uses) advances the
//     lengths;
//   * launched with programmatic dependent launch: a CTA makes its aligned
//     plan before it waits for the previous grid, and lets the next grid
//     launch as soon as its own wait is over.  (An L2 prefetch of the CTA's
//     pages before the wait was measured and removed: it cost 1.1 us at B=1
//     and 18 % at B=16, where the ranges exceed L2.)
#include "common.cuh"

namespace hq {
namespace {

// NC consumer warps with 2 stages each, one producer warp, one CTA per SM.
// Each stage must have exactly one consumer warp: a parity wait on an mbarrier
// only tells the current phase from the one before it, so a warp that reached a
// stage while another warp's earlier tile there had not landed yet would see the
// older completed phase and consume the wrong data.  With NSTAGES = 2 NC,
// stage s belongs to warp s % NC.
#ifndef HQ_DECODE_NC
#define HQ_DECODE_NC 11
#endif
constexpr int NC = HQ_DECODE_NC;
constexpr int NSTAGES = 2 * NC;
constexpr int NTHREADS = (NC + 1) * 32;
constexpr int FT = 16;                         // rows per FP16 tile
constexpr int FSTRIDE = 256;                   // bytes per FP16 row in shared memory (one contiguous copy)
constexpr int OFF_FV = FT * FSTRIDE;           // V rows of an FP16 tile
constexpr int STAGE_BYTES = 10368;             // max(10256, 2 * 16 * 256 = 8192), 128-aligned
constexpr int PART_FLOATS = 16 + 8 * D;        // m[8], l[8], O[8][128]
constexpr int MAX_UNITS = 2048;                // (b, kv head) units per call
constexpr int MAXSEG = 88;                     // segments (units) one CTA's range can touch
constexpr int PHANTOM_DIV = 32;                // phantom weight per unit = ceil(tiles / (CTAs x 32))
constexpr int MIN_TILES = 4;                   // at least this many tiles per CTA
constexpr int MAX_CTAS = 160;                  // one CTA per SM, at most this many (the unit merge keeps one weight per CTA in a stage)
constexpr int SCAN_PER = (MAX_UNITS + NTHREADS - 1) / NTHREADS;  // units per thread in the scan
static_assert(HQ_PAGE_SUBBYTES(4, 4) + 16 <= STAGE_BYTES && HQ_PAGE_SUBBYTES(8, 8) + 16 <= STAGE_BYTES &&
                  HQ_PAGE_SUBBYTES(4, 2) + 16 <= STAGE_BYTES && HQ_PAGE_SUBBYTES(2, 4) + 16 <= STAGE_BYTES,
              "a packed stage holds one sub-page and the page's bitmap words");
static_assert(PART_FLOATS * 4 <= STAGE_BYTES, "a warp state fits in one stage");

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

// ------------------------------------------------------------------ work decomposition

// One unit's lengths and tile counts (from its sequence's state row).
struct UnitGeo {
  int n_packed, n_vl, T;
  int NP, NV, NF, NT;   // packed tiles, VL tiles, FP16 tiles (VL + ring + new token), all
};

__device__ __forceinline__ UnitGeo unit_geo(int n_packed, int n_vl, int T, int R, int pr) {
  UnitGeo g;
  g.n_packed = n_packed;
  g.n_vl = n_vl;
  g.T = T;
  g.NP = (n_packed + pr - 1) / pr;  // packed tiles: sub-pages of pr positions
  g.NV = (n_vl + FT - 1) / FT;
  g.NF = g.NV + R / FT + 1;
  g.NT = g.NP + g.NF;
  return g;
}

// A sequence takes no step when its staging area is full or T reached cap.
__device__ __forceinline__ bool refused(const hq_cache& c, int T, int n_packed) {
  return T - n_packed >= c.W + HQ_STAGE || T >= c.cap;
}

// Number of FP16 tiles among the unit's first k tiles (FP16 tiles spread evenly).
__device__ __forceinline__ int fp16_before(const UnitGeo& g, int k) {
  return static_cast<int>((static_cast<long long>(k) * g.NF) / g.NT);
}

// 16-bit mask of the valid rows of FP16 tile j (VL tiles, then ring tiles, then the new token)
__device__ __forceinline__ uint32_t fp16_valid(const UnitGeo& g, int j, int R) {
  if (j < g.NV) {
    const int n = min(FT, g.n_vl - j * FT);
    return n >= FT ? 0xFFFFu : ((1u << n) - 1u);
  }
  const int r = j - g.NV;
  if (r == R / FT) return 1u;  // the new token
  // ring slot s holds position p = n_packed + ((s - n_packed) mod R); valid iff p < T
  const int base = g.n_packed % R;
  uint32_t m = 0;
#pragma unroll 4
  for (int i = 0; i < FT; ++i) {
    int off = FT * r + i - base;
    off += off < 0 ? R : 0;
    m |= (g.n_packed + off < g.T ? 1u : 0u) << i;
  }
  return m;
}

// A CTA's share of one unit: CTA-local tiles [a, b), which the CTA runs packed
// ones first (pages p0 .. p0 + npk - 1), then FP16 ones (f0 ..): a warp that
// gets one tile more than the others then gets a cheap FP16 tile.
struct Seg {
  int u, a, b, p0, npk, f0, first_cta, ncta;
};

// CTA-local tile i of segment sg: the packed tile index (>= 0), or -(FP16 tile index) - 1.
__device__ __forceinline__ int seg_tile(const Seg& sg, int i) {
  const int j = i - sg.a;
  return j < sg.npk ? sg.p0 + j : -(sg.f0 + j - sg.npk) - 1;
}

// The CTA's range and segments (shared memory), built by all NTHREADS threads.
struct Plan {
  int nseg, ntile, u0;
  long long X, Wt, w0, w1;
  int ceff;
  Seg seg[MAXSEG];
};

__device__ __forceinline__ void read_len(const hq_cache& c, int b, bool stale, int& T, int& np, int& nv) {
  const int32_t* st = state_row(c, b);
  if (stale) {
    T = *reinterpret_cast<volatile const int*>(st + HQ_STATE_T);
    np = min(max(*reinterpret_cast<volatile const int*>(st + HQ_STATE_NPACKED), 0), c.cap);
    nv = min(max(*reinterpret_cast<volatile const int*>(st + HQ_STATE_NVL), 0), c.vl_cap);
  } else {
    T = st[HQ_STATE_T];
    np = st[HQ_STATE_NPACKED];
    nv = st[HQ_STATE_NVL];
  }
}

// Few units (4 CTAs or more per unit): every unit gets its own CTAs, in
// proportion to its tiles (at least one, at most one tile per consumer warp),
// and each of them an even share of the unit's packed tiles and of its FP16
// tiles, so a CTA has one segment and no range crosses a unit.  The last
// ALIGNED_SPARE CTAs get no work: they are the ones the block scheduler starts
// last (their SMs free up last), so no unit waits for a late CTA.
constexpr int ALIGNED_SPARE = 12;
constexpr int ALIGNED_MAX_UNITS = MAX_CTAS / 4;

// The lengths an aligned plan was made from: per sequence (n_packed, n_vl,
// takes a step), per unit (packed tiles, FP16 tiles).
struct AlignedSnap {
  int np[ALIGNED_MAX_UNITS], nv[ALIGNED_MAX_UNITS], go[ALIGNED_MAX_UNITS];
  int NP[ALIGNED_MAX_UNITS], NF[ALIGNED_MAX_UNITS];
};

// One thread per unit (U <= ALIGNED_MAX_UNITS) records the lengths.
__device__ __forceinline__ void aligned_snapshot(const hq_cache& c, int R, AlignedSnap& sn, bool stale) {
  const int U = c.B * c.Hkv;
  const int tid = threadIdx.x;
  if (tid < U) {
    int T, np, nv;
    read_len(c, tid / c.Hkv, stale, T, np, nv);
    const bool go = !refused(c, T, np);
    const UnitGeo g = unit_geo(np, nv, T, R, page_geo(c).pr);
    sn.NP[tid] = go ? g.NP : 0;
    sn.NF[tid] = go ? g.NF : 0;
    if (tid % c.Hkv == 0) {
      const int b = tid / c.Hkv;
      sn.np[b] = np;
      sn.nv[b] = nv;
      sn.go[b] = go;
    }
  }
}

// True (block-wide) when a sequence's lengths differ from the snapshot in a
// way that changes the plan (n_packed, n_vl, or whether it takes a step).
__device__ __forceinline__ bool aligned_changed(const hq_cache& c, const AlignedSnap& sn) {
  bool ch = false;
  if (static_cast<int>(threadIdx.x) < c.B) {
    int T, np, nv;
    read_len(c, threadIdx.x, false, T, np, nv);
    ch = np != sn.np[threadIdx.x] || nv != sn.nv[threadIdx.x] || (!refused(c, T, np)) != (sn.go[threadIdx.x] != 0);
  }
  return __syncthreads_or(ch) != 0;
}

// Thread 0: the split table and this CTA's segment.
__device__ __forceinline__ void aligned_assign(const hq_cache& c, Plan& p, const AlignedSnap& sn) {
  const int U = c.B * c.Hkv;
  long long N = 0;
  for (int u = 0; u < U; ++u) N += sn.NP[u] + sn.NF[u];
  const int C = static_cast<int>(gridDim.x) - (static_cast<int>(gridDim.x) >= 4 * U + ALIGNED_SPARE ? ALIGNED_SPARE : 0);
  const long long C2 = C - U;  // CTAs to share out beyond one per unit
  int at = 0, mine = -1, j = 0, S = 1;
  for (int u = 0; u < U; ++u) {
    const int nt = sn.NP[u] + sn.NF[u];
    const int Su = nt == 0 ? 0
                           : min(1 + static_cast<int>(N > 0 ? (static_cast<long long>(nt) * C2) / N : 0), (nt + NC - 1) / NC);
    if (static_cast<int>(blockIdx.x) >= at && static_cast<int>(blockIdx.x) < at + Su) {
      mine = u;
      j = blockIdx.x - at;
      S = Su;
      p.seg[0].first_cta = at;
      p.seg[0].ncta = Su;
    }
    at += Su;
  }
  p.ceff = at;
  p.nseg = 0;
  p.ntile = 0;
  if (mine >= 0) {
    const int NP = sn.NP[mine], NF = sn.NF[mine];
    Seg& sg = p.seg[0];
    sg.u = mine;
    sg.p0 = (j * NP) / S;
    sg.npk = ((j + 1) * NP) / S - sg.p0;
    sg.f0 = (j * NF) / S;
    const int nf = ((j + 1) * NF) / S - sg.f0;
    sg.a = 0;
    sg.b = sg.npk + nf;
    if (sg.b > 0) {
      p.nseg = 1;
      p.ntile = sg.b;
    }
  }
}

// Cut the batch's tile lists into ranges and record this CTA's segments.
// `stale`: state read with volatile loads (it may be one step old).  `red`
// is scratch for NTHREADS / 32 ints.
__device__ __noinline__ void make_plan(const hq_cache& c, int R, Plan& p, int* red, bool stale) {
  const int U = c.B * c.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < MAXSEG) p.seg[tid].u = -1;
  // tile counts of this thread's units (sequences that take no step: none)
  int nt[SCAN_PER];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < SCAN_PER; ++i) {
    const int u = tid * SCAN_PER + i;
    nt[i] = 0;
    if (u < U) {
      int T, np, nv;
      read_len(c, u / c.Hkv, stale, T, np, nv);
      if (!refused(c, T, np)) nt[i] = unit_geo(np, nv, T, R, page_geo(c).pr).NT;
    }
    sum += nt[i];
  }
  // block-wide exclusive scan of the per-thread sums
  int x = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  if (tid == 0) {
    p.nseg = 0;
    p.u0 = -1;
  }
  __syncthreads();
  int before = 0, total = 0;
  for (int w = 0; w < NTHREADS / 32; ++w) {
    const int v = red[w];
    before += w < warp ? v : 0;
    total += v;
  }
  const int excl = before + x - sum;  // tiles of all units before this thread's first unit
  if (tid == 0) {
    // ceff CTAs share the work (at least U / 48 of them); a phantom weight X per
    // unit bounds the units one range can touch by N / (ceff X) + U / ceff + 2
    // <= 32 + 48 + 2 < MAXSEG
    const long long N = total;
    const long long ceff = min(static_cast<long long>(gridDim.x),
                               max(max(1ll, (N + MIN_TILES - 1) / MIN_TILES), static_cast<long long>((U + 47) / 48)));
    const long long X = max(1ll, (N + ceff * PHANTOM_DIV - 1) / (ceff * PHANTOM_DIV));
    const long long Wt = N + static_cast<long long>(U) * X;
    p.ceff = static_cast<int>(ceff);
    p.X = X;
    p.Wt = Wt;
    p.w0 = (static_cast<long long>(blockIdx.x) * Wt) / ceff;
    p.w1 = (static_cast<long long>(blockIdx.x + 1) * Wt) / ceff;
  }
  __syncthreads();
  const long long X = p.X, Wt = p.Wt, w0 = p.w0, w1 = p.w1;
  const int ceff = p.ceff;
  // the unit holding w0: unit u spans weights [S_u, S_u + X + NT_u), S_u = tiles before + u X
  int tb = excl;
#pragma unroll
  for (int i = 0; i < SCAN_PER; ++i) {
    const int u = tid * SCAN_PER + i;
    if (u < U) {
      const long long S = tb + static_cast<long long>(u) * X;
      if (S <= w0 && w0 < S + X + nt[i]) p.u0 = u;
    }
    tb += nt[i];
  }
  __syncthreads();
  const int u0 = p.u0;
  // every unit of [u0, u0 + MAXSEG) that holds tiles of this CTA's range becomes a segment
  tb = excl;
#pragma unroll
  for (int i = 0; i < SCAN_PER; ++i) {
    const int u = tid * SCAN_PER + i;
    if (u < U && u >= u0 && u0 >= 0 && nt[i] > 0) {
      const long long S = tb + static_cast<long long>(u) * X + X;  // first tile's weight
      const long long lo = max(S, w0), hi = min(S + nt[i], w1);
      if (lo < hi) {
        if (u - u0 < MAXSEG) {
          int T, np, nv;
          read_len(c, u / c.Hkv, stale, T, np, nv);
          const UnitGeo g = unit_geo(np, nv, T, R, page_geo(c).pr);
          Seg& s = p.seg[u - u0];
          const int k0 = static_cast<int>(lo - S), k1 = static_cast<int>(hi - S);
          s.u = u;
          s.b = k1 - k0;  // a count for now; CTA-local positions are set below
          s.f0 = fp16_before(g, k0);
          s.p0 = k0 - s.f0;
          s.npk = (k1 - fp16_before(g, k1)) - s.p0;
          auto cta_of = [&](long long w) { return static_cast<int>(((w + 1) * ceff - 1) / Wt); };
          s.first_cta = cta_of(S);
          s.ncta = cta_of(S + nt[i] - 1) - s.first_cta + 1;
          atomicMax(&p.nseg, u - u0 + 1);
        } else {
          set_err(state_row(c, 0), HQ_DEVERR_TIMEOUT);  // never expected: the phantom weight bounds the count
        }
      }
    }
    tb += nt[i];
  }
  __syncthreads();
  if (tid == 0) {
    // CTA-local tile numbering: segments back to back, empty slots skipped
    int at = 0, k = 0;
    for (int i = 0; i < p.nseg; ++i) {
      Seg t = p.seg[i];
      if (t.u != u0 + i || t.b <= 0) continue;
      const int n = t.b;
      t.a = at;
      t.b = at + n;
      at += n;
      p.seg[k++] = t;
    }
    p.nseg = blockIdx.x < ceff ? k : 0;
    p.ntile = blockIdx.x < ceff ? at : 0;
  }
  __syncthreads();
}

struct WarpState {
  float m[2], l[2];
  float o[8][4];
};

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
  // the running max only has to move when some logit exceeds it by more than
  // LAZY_MAX: one vote on the thread-local maxima decides, and the reduction
  // over the query column's 8 lanes runs only then (rarely after the first tile)
  if (__any_sync(0xffffffffu, mx0 > ws.m[0] + LAZY_MAX || mx1 > ws.m[1] + LAZY_MAX)) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const bool up0 = mx0 > ws.m[0] + LAZY_MAX, up1 = mx1 > ws.m[1] + LAZY_MAX;
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

// ------------------------------------------------------------------ packed tiles of any code width
//
// A packed tile is one sub-page of PR = HQ_PAGE_SUBPOS(KB, VB) positions (64,
// or 32 for K8V8) copied verbatim into the stage, followed by the page's two
// bitmap words at the stage offset SUB = HQ_PAGE_SUBBYTES(KB, VB).  Inside the
// stage: K codes [PR][16 KB], V codes [PR][16 VB], K (scale | zero << 16) words
// [PR][4], V words [PR][4].

// 2-bit codes: value j (bits 2j, 2j+1) of the bytes at bits 0..7 and 16..23 of x
// -> (1024 + 4^j n) in both halves, scaled back by 4^-j and shifted by -1024 4^-j
// (exact: 1024 + 4^j n < 2048 keeps unit spacing).
__device__ __forceinline__ uint32_t two_bit(uint32_t x, int j) {
  const uint32_t m = and_or(x, 0x00030003u << (2 * j), MAGIC);
  if (j == 0) return hsub2_u(m, H2_1024);
  const uint32_t sc = j == 1 ? 0x34003400u : (j == 2 ? 0x2C002C00u : 0x24002400u);   // 1/4, 1/16, 1/64
  const uint32_t off = j == 1 ? 0xDC00DC00u : (j == 2 ? 0xD400D400u : 0xCC00CC00u);  // -256, -64, -16
  return hfma2_u(m, sc, off);
}
// 8-bit codes: bytes b0 (bits 0..7) and b1 (bits 16..23) of p -> (b0, b1) as fp16
__device__ __forceinline__ uint32_t eight_bit(uint32_t p) { return hsub2_u(and_or(p, 0x00FF00FFu, MAGIC), H2_1024); }

// Q^T fragments of the thread's 32 dims in the order the K codes of width KB
// dequantise to (k-step kk: b0 = Q at the dims of a0, b1 = Q at the dims of a2).
template <int KB>
__device__ __forceinline__ void q_frags(const uint4 (&u)[4], uint32_t (&qf)[8][2]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (KB == 4) {  // word i, byte h: (d 8i+2h, 8i+2h+4) and (8i+2h+1, 8i+2h+5)
      qf[2 * i][0] = prmt(u[i].x, u[i].z, 0x5410);
      qf[2 * i][1] = prmt(u[i].x, u[i].z, 0x7632);
      qf[2 * i + 1][0] = prmt(u[i].y, u[i].w, 0x5410);
      qf[2 * i + 1][1] = prmt(u[i].y, u[i].w, 0x7632);
    } else if (KB == 8) {  // word kk: (d 4kk, 4kk+1) and (4kk+2, 4kk+3)
      qf[2 * i][0] = u[i].x;
      qf[2 * i][1] = u[i].y;
      qf[2 * i + 1][0] = u[i].z;
      qf[2 * i + 1][1] = u[i].w;
    }
  }
  if (KB == 2) {  // k-step kk = 4 w + j: (d 16w+j, 16w+8+j) and (16w+4+j, 16w+12+j)
    const uint32_t h[16] = {u[0].x, u[0].y, u[0].z, u[0].w, u[1].x, u[1].y, u[1].z, u[1].w,
                            u[2].x, u[2].y, u[2].z, u[2].w, u[3].x, u[3].y, u[3].z, u[3].w};
#pragma unroll
    for (int w = 0; w < 2; ++w)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int b = 8 * w;  // half2 words of dims 16w ..
        const uint32_t sel = (j & 1) ? 0x7632 : 0x5410;
        qf[4 * w + j][0] = prmt(h[b + (j >> 1)], h[b + 4 + (j >> 1)], sel);
        qf[4 * w + j][1] = prmt(h[b + 2 + (j >> 1)], h[b + 6 + (j >> 1)], sel);
      }
  }
}

// The A-fragment halves of k-step kk for one key row whose group-t codes are
// in w[] (4 KB bytes): lo = the dims of a0 (or a1), hi = those of a2 (or a3),
// dequantised with the group's (scale, zero) pair s2, z2.
template <int KB>
__device__ __forceinline__ void k_step(const uint32_t (&w)[KB], int kk, uint32_t s2, uint32_t z2, uint32_t& lo,
                                       uint32_t& hi) {
  if (KB == 4) {
    const uint32_t x = w[kk >> 1] >> (8 * (kk & 1));
    lo = hfma2_u(nib_lo(x), s2, z2);
    hi = hfma2_u(nib_hi(x), s2, z2);
  } else if (KB == 8) {
    lo = hfma2_u(eight_bit(prmt(w[kk], 0u, 0x4140)), s2, z2);
    hi = hfma2_u(eight_bit(prmt(w[kk], 0u, 0x4342)), s2, z2);
  } else {
    const uint32_t x = w[kk >> 2];
    lo = hfma2_u(two_bit(x, kk & 3), s2, z2);
    hi = hfma2_u(two_bit(x >> 8, kk & 3), s2, z2);
  }
}

// one packed tile by one warp: S^T = K^ . Q^T for its 16-key blocks, one
// online-softmax step for all of them, O^T += V^T . P^T
template <int KB, int VB>
__device__ __forceinline__ void packed_tile(WarpState& ws, const uint8_t* st, const uint32_t (&qf)[8][2], int tile, int n_packed,
                                            float qscale, int g, int t) {
  constexpr int PR = HQ_PAGE_SUBPOS(KB, VB), NMT = PR / 16;
  constexpr int OFFV = PR * 16 * KB, OFFKS = PR * 16 * (KB + VB), OFFVS = OFFKS + PR * 16, OFFM = HQ_PAGE_SUBBYTES(KB, VB);
  const uint8_t* kc = st;
  const uint8_t* vc = st + OFFV;
  const uint32_t* ks = reinterpret_cast<const uint32_t*>(st + OFFKS);
  const uint32_t* vs = reinterpret_cast<const uint32_t*>(st + OFFVS);
  const uint32_t* mk = reinterpret_cast<const uint32_t*>(st + OFFM);
  const int base = tile * PR;
  const int prow0 = base & 63;  // first page row of the tile
  const bool full = base + PR <= n_packed;
  const int pa = pi_pk(g), pbk = pi_pk(g + 8);
  // additive score bias of this thread's key rows: -inf beyond n_packed or on
  // a vertical line (its FP16 row is read instead), else 0
  float bias[NMT][2];
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt) {
    const int ra = 16 * mt + pa, rb = 16 * mt + pbk;
    const int qa = prow0 + ra, qb = prow0 + rb;
    const bool va = (full || base + ra < n_packed) && !((mk[qa >> 5] >> (qa & 31)) & 1u);
    const bool vb = (full || base + rb < n_packed) && !((mk[qb >> 5] >> (qb & 31)) & 1u);
    bias[mt][0] = va ? 0.f : -INFINITY;
    bias[mt][1] = vb ? 0.f : -INFINITY;
  }

  float s[NMT][4];
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt) {
    const int ra = 16 * mt + pa, rb = 16 * mt + pbk;
    uint32_t wa[KB], wb[KB];  // group t of rows a and b: 4 KB bytes = KB words each
#pragma unroll
    for (int i = 0; i < KB / 4; ++i) {
      const uint4 x = *reinterpret_cast<const uint4*>(kc + ra * 16 * KB + 4 * KB * t + 16 * i);
      const uint4 y = *reinterpret_cast<const uint4*>(kc + rb * 16 * KB + 4 * KB * t + 16 * i);
      wa[4 * i] = x.x; wa[4 * i + 1] = x.y; wa[4 * i + 2] = x.z; wa[4 * i + 3] = x.w;
      wb[4 * i] = y.x; wb[4 * i + 1] = y.y; wb[4 * i + 2] = y.z; wb[4 * i + 3] = y.w;
    }
    if (KB == 2) {
      const uint2 x = *reinterpret_cast<const uint2*>(kc + ra * 32 + 8 * t);
      const uint2 y = *reinterpret_cast<const uint2*>(kc + rb * 32 + 8 * t);
      wa[0] = x.x; wa[1] = x.y;
      wb[0] = y.x; wb[1] = y.y;
    }
    const uint32_t za = ks[ra * 4 + t], zb = ks[rb * 4 + t];
    const uint32_t sa2 = prmt(za, za, 0x1010), za2 = prmt(za, za, 0x3232);
    const uint32_t sb2 = prmt(zb, zb, 0x1010), zb2 = prmt(zb, zb, 0x3232);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a0, a1, a2, a3;
      k_step<KB>(wa, kk, sa2, za2, a0, a2);
      k_step<KB>(wb, kk, sb2, zb2, a1, a3);
      mma16816(acc, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
    }
    s[mt][0] = fmaf(acc[0], qscale, bias[mt][0]);
    s[mt][1] = fmaf(acc[1], qscale, bias[mt][0]);
    s[mt][2] = fmaf(acc[2], qscale, bias[mt][1]);
    s[mt][3] = fmaf(acc[3], qscale, bias[mt][1]);
  }
  uint32_t pb[NMT][2];
  softmax_update<NMT>(ws, s, pb);

#pragma unroll
  for (int mt = 0; mt < NMT; ++mt) {
    const int r0 = 16 * mt + pi_pk(2 * t), r1 = 16 * mt + pi_pk(2 * t + 1);
    const int r2 = 16 * mt + pi_pk(2 * t + 8), r3 = 16 * mt + pi_pk(2 * t + 9);
    const int grp = g >> 1;
    const uint32_t z0 = vs[r0 * 4 + grp], z1 = vs[r1 * 4 + grp], z2 = vs[r2 * 4 + grp], z3 = vs[r3 * 4 + grp];
    const uint32_t s01 = prmt(z0, z1, 0x5410), o01 = prmt(z0, z1, 0x7632);
    const uint32_t s23 = prmt(z2, z3, 0x5410), o23 = prmt(z2, z3, 0x7632);
    uint32_t keep_ab = 0xFFFFFFFFu, keep_cd = 0xFFFFFFFFu;
    if (!full) {  // rows past n_packed may hold stale records: zero them out of P.V
      keep_ab = (base + r0 < n_packed ? 0x0000FFFFu : 0u) | (base + r1 < n_packed ? 0xFFFF0000u : 0u);
      keep_cd = (base + r2 < n_packed ? 0x0000FFFFu : 0u) | (base + r3 < n_packed ? 0xFFFF0000u : 0u);
    }
    // a0 / a1: keys (r0, r1) at dims 16g + 2m and 16g + 2m + 1; a2 / a3: keys (r2, r3)
    uint32_t A[8][4];
    if (VB == 4) {
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
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const uint32_t yab = xab[m >> 1] >> (8 * (m & 1));
        const uint32_t ycd = xcd[m >> 1] >> (8 * (m & 1));
        A[m][0] = hfma2_u(nib_lo(yab), s01, o01);
        A[m][1] = hfma2_u(nib_hi(yab), s01, o01);
        A[m][2] = hfma2_u(nib_lo(ycd), s23, o23);
        A[m][3] = hfma2_u(nib_hi(ycd), s23, o23);
      }
    } else if (VB == 8) {
      // 16 bytes per row (dims 16g .. 16g + 15): byte d of key r0 beside byte d of key r1
      const uint4 u0 = *reinterpret_cast<const uint4*>(vc + r0 * 128 + 16 * g);
      const uint4 u1 = *reinterpret_cast<const uint4*>(vc + r1 * 128 + 16 * g);
      const uint4 u2 = *reinterpret_cast<const uint4*>(vc + r2 * 128 + 16 * g);
      const uint4 u3 = *reinterpret_cast<const uint4*>(vc + r3 * 128 + 16 * g);
      const uint32_t q0[4] = {u0.x, u0.y, u0.z, u0.w}, q1[4] = {u1.x, u1.y, u1.z, u1.w};
      const uint32_t q2[4] = {u2.x, u2.y, u2.z, u2.w}, q3[4] = {u3.x, u3.y, u3.z, u3.w};
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int b = 2 * (m & 1);  // byte of dim 2m in word m / 2
        const uint32_t sl = b | (b << 4) | ((4 + b) << 8) | ((4 + b) << 12);
        const uint32_t sh = (b + 1) | ((b + 1) << 4) | ((5 + b) << 8) | ((5 + b) << 12);
        A[m][0] = hfma2_u(eight_bit(prmt(q0[m >> 1], q1[m >> 1], sl)), s01, o01);
        A[m][1] = hfma2_u(eight_bit(prmt(q0[m >> 1], q1[m >> 1], sh)), s01, o01);
        A[m][2] = hfma2_u(eight_bit(prmt(q2[m >> 1], q3[m >> 1], sl)), s23, o23);
        A[m][3] = hfma2_u(eight_bit(prmt(q2[m >> 1], q3[m >> 1], sh)), s23, o23);
      }
    } else {
      // 4 bytes per row (dims 16g .. 16g + 15, byte k = dims 4k .. 4k + 3)
      const uint32_t w0 = reinterpret_cast<const uint32_t*>(vc + r0 * 32)[g];
      const uint32_t w1 = reinterpret_cast<const uint32_t*>(vc + r1 * 32)[g];
      const uint32_t w2 = reinterpret_cast<const uint32_t*>(vc + r2 * 32)[g];
      const uint32_t w3 = reinterpret_cast<const uint32_t*>(vc + r3 * 32)[g];
      const uint32_t xab[2] = {prmt(w0, w1, 0x5410), prmt(w0, w1, 0x7632)};  // dims 0..7, 8..15 of both keys
      const uint32_t xcd[2] = {prmt(w2, w3, 0x5410), prmt(w2, w3, 0x7632)};
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const uint32_t yab = xab[m >> 2] >> (8 * ((m >> 1) & 1));
        const uint32_t ycd = xcd[m >> 2] >> (8 * ((m >> 1) & 1));
        const int j = 2 * (m & 1);
        A[m][0] = hfma2_u(two_bit(yab, j), s01, o01);
        A[m][1] = hfma2_u(two_bit(yab, j + 1), s01, o01);
        A[m][2] = hfma2_u(two_bit(ycd, j), s23, o23);
        A[m][3] = hfma2_u(two_bit(ycd, j + 1), s23, o23);
      }
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      uint32_t a0 = A[m][0], a1 = A[m][1], a2 = A[m][2], a3 = A[m][3];
      if (!full) {
        a0 &= keep_ab; a1 &= keep_ab;
        a2 &= keep_cd; a3 &= keep_cd;
      }
      mma16816(ws.o[m], a0, a1, a2, a3, pb[mt][0], pb[mt][1]);
    }
  }
}

// one FP16 tile (16 rows at FSTRIDE) by one warp; bit r of `valid` marks row r as real
template <int KB>
__device__ __forceinline__ void fp16_tile(WarpState& ws, const uint8_t* st, const uint32_t (&qf)[8][2], uint32_t valid,
                                          float qscale, int g, int t) {
  const uint8_t* kb = st;
  const uint8_t* vb = st + OFF_FV;
  const int ra = pi_fp(g), rb = pi_fp(g + 8);
  const uint8_t* ka = kb + ra * FSTRIDE + 64 * t;  // the thread's 32 dims of key rows a and b
  const uint8_t* kbr = kb + rb * FSTRIDE + 64 * t;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  // the K A-fragments follow the dim order of the Q fragments (q_frags<KB>)
  if (KB == 2) {
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const uint4 a0 = *reinterpret_cast<const uint4*>(ka + 32 * w), a1 = *reinterpret_cast<const uint4*>(ka + 32 * w + 16);
      const uint4 b0 = *reinterpret_cast<const uint4*>(kbr + 32 * w), b1 = *reinterpret_cast<const uint4*>(kbr + 32 * w + 16);
      const uint32_t ha[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const uint32_t hb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {  // k-step 4w + j: (d 16w+j, 16w+8+j) and (16w+4+j, 16w+12+j)
        const uint32_t sel = (j & 1) ? 0x7632 : 0x5410;
        const int h = j >> 1;
        mma16816(acc, prmt(ha[h], ha[4 + h], sel), prmt(hb[h], hb[4 + h], sel), prmt(ha[2 + h], ha[6 + h], sel),
                 prmt(hb[2 + h], hb[6 + h], sel), qf[4 * w + j][0], qf[4 * w + j][1]);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 ua = *reinterpret_cast<const uint4*>(ka + 16 * i);
      const uint4 ub = *reinterpret_cast<const uint4*>(kbr + 16 * i);
      if (KB == 4) {
        // k-step 2i: (d0,d4) and (d1,d5); k-step 2i+1: (d2,d6) and (d3,d7)
        mma16816(acc, prmt(ua.x, ua.z, 0x5410), prmt(ub.x, ub.z, 0x5410), prmt(ua.x, ua.z, 0x7632),
                 prmt(ub.x, ub.z, 0x7632), qf[2 * i][0], qf[2 * i][1]);
        mma16816(acc, prmt(ua.y, ua.w, 0x5410), prmt(ub.y, ub.w, 0x5410), prmt(ua.y, ua.w, 0x7632),
                 prmt(ub.y, ub.w, 0x7632), qf[2 * i + 1][0], qf[2 * i + 1][1]);
      } else {
        // k-step 2i: (d0,d1) and (d2,d3); k-step 2i+1: (d4,d5) and (d6,d7)
        mma16816(acc, ua.x, ub.x, ua.y, ub.y, qf[2 * i][0], qf[2 * i][1]);
        mma16816(acc, ua.z, ub.z, ua.w, ub.w, qf[2 * i + 1][0], qf[2 * i + 1][1]);
      }
    }
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


// The last CTA to take its grid ticket advances every stepping sequence's T
// (and its count of buffered queries).  Every CTA takes its ticket only after
// it has read all the lengths it uses, so no CTA sees a T of the next step;
// the appends of the units need no ordering with this (they were placed from
// the T each CTA read at its start).
__device__ __forceinline__ void advance_lengths(const hq_cache& c, int tid, int nthr, unsigned int* tickets) {
  for (int b = tid; b < c.B; b += nthr) {
    int32_t* st = state_row(c, b);
    const int T = st[HQ_STATE_T];
    if (!refused(c, T, st[HQ_STATE_NPACKED])) {
      st[HQ_STATE_T] = T + 1;
      st[HQ_STATE_NQ] = min(st[HQ_STATE_NQ] + 1, HQ_QBUF);
    }
  }
  if (tid == 0) tickets[0] = 0u;
}

// Load this unit's Q^T fragments (the G query heads of kv head kvh of sequence b,
// in the dim order the K codes dequantise to: thread t covers dims 32t .. 32t+31);
// columns >= G are zero.
template <int KB>
__device__ __forceinline__ void load_q(const hq_cache& c, const uint16_t* __restrict__ q, int b, int kvh, int G, int g,
                                       int t, uint32_t (&qf)[8][2]) {
  if (g < G) {
    const uint4* qp = reinterpret_cast<const uint4*>(q + (static_cast<size_t>(b) * c.Hq + kvh * G + g) * D + 32 * t);
    const uint4 u[4] = {qp[0], qp[1], qp[2], qp[3]};
    q_frags<KB>(u, qf);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) qf[j][0] = qf[j][1] = 0u;
  }
}

__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, %0;" ::"r"(NC * 32) : "memory"); }

__device__ __forceinline__ UnitGeo geo_of_unit(const hq_cache& c, int u, int R) {
  const int32_t* st = state_row(c, u / c.Hkv);
  return unit_geo(st[HQ_STATE_NPACKED], st[HQ_STATE_NVL], st[HQ_STATE_T], R, page_geo(c).pr);
}

// Source of FP16 tile j of unit bh (K rows, V rows, bytes per half)
__device__ __forceinline__ void fp16_src(const hq_cache& c, const UnitGeo& g, int bh, int j, int R,
                                         const uint16_t* k_new, const uint16_t* v_new, const uint16_t*& ks,
                                         const uint16_t*& vs, uint32_t& bytes) {
  if (j < g.NV) {
    const size_t off = (static_cast<size_t>(bh) * c.vl_cap + j * FT) * D;
    ks = c.kf + off;
    vs = c.vf + off;
    bytes = FT * 2 * D;
  } else if (j - g.NV < R / FT) {
    const size_t off = (static_cast<size_t>(bh) * R + (j - g.NV) * FT) * D;
    ks = c.kr + off;
    vs = c.vr + off;
    bytes = FT * 2 * D;
  } else {
    ks = k_new + static_cast<size_t>(bh) * D;
    vs = v_new + static_cast<size_t>(bh) * D;
    bytes = 2 * D;
  }
}

// The end of a segment, on the consumer warps: merge the warp states held in
// their stages into the segment's partial, take the unit's ticket (and, with the
// CTA's last segment, its grid ticket), and in the unit's last CTA merge the
// unit's partials, write its output and append its new token and queries.
__device__ __forceinline__ void segment_epilogue(const hq_cache& c, const uint16_t* __restrict__ q,
                                              const uint16_t* __restrict__ k_new, const uint16_t* __restrict__ v_new,
                                              uint16_t* __restrict__ out, float* __restrict__ parts,
                                              unsigned int* __restrict__ tickets, int lse_ok, uint8_t* smem, int* s_held,
                                              int* s_last_p, int* s_glast_p, const Seg sg, const UnitGeo ug, int si,
                                              int nseg) {
  const int G = c.Hq / c.Hkv;
  const int R = ring_len(c.W);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NTHR = NC * 32;
  const int u = sg.u, b = u / c.Hkv, kvh = u % c.Hkv;
  int& s_last = *s_last_p;
  int& s_glast = *s_glast_p;
  consumer_bar();  // (A) warp states visible
  // ------------------------------------------------------------ CTA merge -> segment partial
  // each thread owns 4 dims of one query and weighs the warp states itself
  const int c_slot = blockIdx.x + u;  // partial slot of (this CTA, unit u)
  float* part = parts + static_cast<size_t>(c_slot) * PART_FLOATS;
  // scratch for the unit merge: a held stage (every segment has a tile, so some
  // warp holds one unless a wait timed out; then stage 0, which stays in bounds)
  int scratch = 0;
  for (int w = NC - 1; w >= 0; --w)
    if (s_held[w] >= 0) scratch = s_held[w];
  for (int it = threadIdx.x; it < 8 * D / 4; it += NTHR) {
    const int qc = (4 * it) / D;
    float mm = -INFINITY;
    for (int w = 0; w < NC; ++w)
      if (s_held[w] >= 0) mm = fmaxf(mm, reinterpret_cast<const float*>(smem + s_held[w] * STAGE_BYTES)[qc]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float ll = 0.f;
    for (int w = 0; w < NC; ++w) {
      if (s_held[w] < 0) continue;
      const float* wsm = reinterpret_cast<const float*>(smem + s_held[w] * STAGE_BYTES);
      const float mw = wsm[qc];
      const float wt = mw == -INFINITY ? 0.f : ex2(mw - mm);
      const float4 o = reinterpret_cast<const float4*>(wsm + 16)[it];
      acc.x = fmaf(wt, o.x, acc.x);
      acc.y = fmaf(wt, o.y, acc.y);
      acc.z = fmaf(wt, o.z, acc.z);
      acc.w = fmaf(wt, o.w, acc.w);
      ll = fmaf(wt, wsm[8 + qc], ll);
    }
    reinterpret_cast<float4*>(part + 16)[it] = acc;
    if ((4 * it) % D == 0) {
      part[qc] = mm;
      part[8 + qc] = ll;
    }
  }
  // the new token's K / V rows and this group's queries, loaded now so that the
  // append after the ticket is stores only (inputs: no ordering concerns)
  const int T = ug.T;
  const int slot = T % R;
  const int bh = u;
  constexpr int APPEND_MAX = (2 + HQ_MAX_GQA) * (D / 8);
  static_assert(APPEND_MAX <= 2 * NC * 32, "at most two 16-byte chunks of the append per consumer thread");
  uint4 app[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
  uint4* app_dst[2] = {nullptr, nullptr};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int e = threadIdx.x + k * NTHR;
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
  // completion ticket of the unit: the barrier orders every thread's partial
  // writes before thread 0's gpu-scope release; the last CTA acquires before
  // the barrier that releases its other threads to read the partials
  // With its last segment the CTA also takes its grid ticket: it has read
  // every length it needs, and the last grid ticket advances the lengths.
  // The two tickets are taken by two threads at once (one round trip to L2).
  consumer_bar();  // (B) partial written, warp states read
  if (threadIdx.x == 0) {
    s_last = atom_add_acq_rel_gpu(&tickets[1 + u], 1u) == static_cast<unsigned>(sg.ncta - 1);
  } else if (threadIdx.x == 32) {
    s_glast = si == nseg - 1 && atom_add_acq_rel_gpu(&tickets[0], 1u) == gridDim.x - 1;
  }
  consumer_bar();  // (C)
  if (s_glast) advance_lengths(c, threadIdx.x, NC * 32, tickets);
  if (s_last) {
    // log-sum-exp merge of the unit's partials (slots first_cta + u ..), in the
    // scratch stage.  The threads split into ngrp groups, each summing the O
    // partials of every ngrp-th CTA for one (query, 4 dims) item; a thread's
    // first PER O loads are issued before the (m, l) of the partials are
    // gathered and weighed, so both round trips to L2 overlap.
    const int S = sg.ncta;
    const float* pb = parts + static_cast<size_t>(sg.first_cta + u) * PART_FLOATS;
    float* sm_m = reinterpret_cast<float*>(smem + scratch * STAGE_BYTES);  // [S][8] weights
    float* sm_inv = sm_m + 8 * S;                                          // [8]
    float4* red4 = reinterpret_cast<float4*>(sm_inv + 8);                  // [ngrp][items]
    constexpr int PER = 12;
    const int items = G * (D / 4);
    const int room = (STAGE_BYTES - 4 * (8 * S + 8)) / (16 * items);      // groups the scratch stage holds
    const int ngrp = max(1, min(min(NTHR / items, S), room));
    const int grp = threadIdx.x / items;
    const int it0 = threadIdx.x - grp * items;
    const bool mine = grp < ngrp;
    const float4* osrc = reinterpret_cast<const float4*>(pb + 16 + (it0 / (D / 4)) * D) + it0 % (D / 4);
    float4 ov[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int sp = grp + j * ngrp;
      ov[j] = (mine && sp < S) ? __ldcg(osrc + sp * (PART_FLOATS / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // partial weights: warp qc weighs query qc's partials, lane s holding s, s + 32, ...
    // (each lane loads its partials' m and l once, in one round trip)
    constexpr int SPL = (MAX_CTAS + 31) / 32;  // partials per lane
    for (int qc = warp; qc < G; qc += NC) {
      float mv[SPL], lv[SPL];
#pragma unroll
      for (int j = 0; j < SPL; ++j) {
        const int sp = lane + 32 * j;
        mv[j] = sp < S ? __ldcg(pb + sp * PART_FLOATS + qc) : -INFINITY;
        lv[j] = sp < S ? __ldcg(pb + sp * PART_FLOATS + 8 + qc) : 0.f;
      }
      float mm = mv[0];
#pragma unroll
      for (int j = 1; j < SPL; ++j) mm = fmaxf(mm, mv[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, o));
      float ll = 0.f;
#pragma unroll
      for (int j = 0; j < SPL; ++j) {
        const int sp = lane + 32 * j;
        if (sp < S) {
          const float w0 = mv[j] == -INFINITY ? 0.f : ex2(mv[j] - mm);
          ll = fmaf(w0, lv[j], ll);
          sm_m[sp * 8 + qc] = w0;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ll += __shfl_xor_sync(0xffffffffu, ll, o);
      if (lane == 0) {
        sm_inv[qc] = ll > 0.f ? 1.0f / ll : 0.f;
        if (c.qlse != nullptr)  // the query's log-sum-exp (base 2), kept for the next reselection
          c.qlse[(static_cast<size_t>(b) * c.Hq + kvh * G + qc) * HQ_QBUF + (T % HQ_QBUF)] =
              lse_ok ? mm + __log2f(ll) : __int_as_float(0x7fc00000);
      }
    }
    consumer_bar();
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
      for (int sp = grp + PER * ngrp; sp < S; sp += ngrp) {  // more than PER partials per group
        const float4 o = __ldcg(osrc + sp * (PART_FLOATS / 4));
        const float w = sm_m[sp * 8 + qc];
        acc.x = fmaf(w, o.x, acc.x);
        acc.y = fmaf(w, o.y, acc.y);
        acc.z = fmaf(w, o.z, acc.z);
        acc.w = fmaf(w, o.w, acc.w);
      }
      red4[grp * items + it0] = acc;
    }
    consumer_bar();
    for (int it = threadIdx.x; it < items; it += NTHR) {
      float4 acc = red4[it];
      for (int g2 = 1; g2 < ngrp; ++g2) {
        const float4 o = red4[g2 * items + it];
        acc.x += o.x;
        acc.y += o.y;
        acc.z += o.z;
        acc.w += o.w;
      }
      const int qc = it / (D / 4), d4 = it % (D / 4);
      const float inv = sm_inv[qc];
      __half2* dst = reinterpret_cast<__half2*>(out + (static_cast<size_t>(b) * c.Hq + kvh * G + qc) * D) + 2 * d4;
      dst[0] = __floats2half2_rn(acc.x * inv, acc.y * inv);
      dst[1] = __floats2half2_rn(acc.z * inv, acc.w * inv);
    }
    // every CTA of this unit has consumed its tiles: append the new token to
    // the ring (slot T % R) and this group's queries to the query buffer
    if (app_dst[0]) *app_dst[0] = app[0];
    if (app_dst[1]) *app_dst[1] = app[1];
    if (threadIdx.x == 0) tickets[1 + u] = 0u;
  }
  // (D) scratch and warp states no longer read: give the held stages back (the
  // generic-proxy writes to them are ordered before the producer's next bulk copy)
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  consumer_bar();
}

template <int KB, int VB>
__global__ void __launch_bounds__(NTHREADS, 1)
decode_kernel(const hq_cache c, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k_new,
              const uint16_t* __restrict__ v_new, uint16_t* __restrict__ out, float qscale,
              float* __restrict__ parts, unsigned int* __restrict__ tickets, int lse_ok) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[NSTAGES], empty[NSTAGES];
  __shared__ Plan plan;
  __shared__ int red[NTHREADS / 32];
  __shared__ int s_timeout;          // a bounded wait gave up somewhere in this CTA
  __shared__ int s_issued[NSTAGES];  // tiles issued into each stage
  __shared__ int s_held[NC];         // stage holding each consumer warp's state at a segment end (-1: none)
  __shared__ int s_last, s_glast;

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
  // the plan: unit-aligned splits for few units (made before the dependency
  // wait on the lengths as they stand, kept after it when they did not
  // change), stream-K ranges for many (made after the wait)
  const bool aligned = c.B * c.Hkv * 4 <= static_cast<int>(gridDim.x);
  __shared__ AlignedSnap snap;
  if (aligned) {
    aligned_snapshot(c, R, snap, true);
    __syncthreads();
    if (threadIdx.x == 0) aligned_assign(c, plan, snap);
    __syncthreads();
  }
  // programmatic dependent launch: everything this kernel reads (the state, the
  // cache, the previous step's appended token) was written by earlier kernels,
  // so wait for them first; then let the next step's grid start launching onto
  // the SMs that free up (it waits here in turn)
  griddep_wait();
  griddep_launch_dependents();
  __syncthreads();  // the stale plan is no longer read
  if (aligned) {
    // the plan made before the wait stands unless a length it used changed
    if (aligned_changed(c, snap)) {
      aligned_snapshot(c, R, snap, false);
      __syncthreads();
      if (threadIdx.x == 0) aligned_assign(c, plan, snap);
      __syncthreads();
    }
  } else {
    make_plan(c, R, plan, red, false);
  }
  if (blockIdx.x == 0) {  // sequences that take no step are flagged (once)
    for (int b = threadIdx.x; b < c.B; b += NTHREADS) {
      int32_t* st = state_row(c, b);
      const int T = st[HQ_STATE_T], np = st[HQ_STATE_NPACKED];
      if (refused(c, T, np)) set_err(st, T >= c.cap ? HQ_DEVERR_CAPACITY : HQ_DEVERR_STAGING_FULL);
    }
  }
  const int ntile = plan.ntile, nseg = plan.nseg;

  if (ntile == 0) {
    // no tiles for this CTA: it only takes its grid ticket
    if (threadIdx.x == 0) s_glast = atom_add_acq_rel_gpu(&tickets[0], 1u) == gridDim.x - 1;
    __syncthreads();
    if (s_glast) advance_lengths(c, threadIdx.x, NTHREADS, tickets);
  } else if (warp == NC) {
    // ---------------------------------------------------------------- producer
    // lane s owns stage s and issues tiles s, s + NSTAGES, s + 2 NSTAGES, ...
    // (1 bulk copy per packed page, 2 per FP16 tile): the initial fill of every
    // stage leaves in one instruction, and a refill waits only for its own stage
    static_assert(NSTAGES <= 32, "one producer lane per stage");
    if (lane < NSTAGES) {
      const int s = lane;
      uint8_t* st = smem + s * STAGE_BYTES;
      int32_t* srow0 = state_row(c, 0);
      int k = 0;   // uses of this stage so far
      int si = 0;  // segment cursor
      UnitGeo ug = geo_of_unit(c, plan.seg[0].u, R);
      for (int i = s; i < ntile; i += NSTAGES, ++k) {
        while (i >= plan.seg[si].b) {
          ++si;
          ug = geo_of_unit(c, plan.seg[si].u, R);
        }
        const Seg sg = plan.seg[si];
        int32_t* srow = state_row(c, sg.u / c.Hkv);
        // the k-th refill waits for the consumer's k-th release (phase k - 1)
        if (k > 0 && !mbar_wait(&empty[s], (k - 1) & 1, srow)) {
          s_timeout = 1;
          break;
        }
        s_issued[s] = k + 1;
        const int tl = seg_tile(sg, i);
        if (tl >= 0) {
          // packed tile tl = sub-page tl % (64 / PR) of page tl / (64 / PR); the
          // page's bitmap words follow the sub-page in the stage
          constexpr int PR = HQ_PAGE_SUBPOS(KB, VB), SUB = HQ_PAGE_SUBBYTES(KB, VB), MOFF = HQ_PAGE_MASK_OFF(KB, VB);
          const uint8_t* page = page_of(c, sg.u, tl * PR);
          mbar_arrive_expect_tx(&full[s], SUB + 16);
          if (PR == 64) {
            bulk_g2s(st, page, SUB + 16, &full[s]);
          } else {
            bulk_g2s(st, page + (tl % (64 / PR)) * SUB, SUB, &full[s]);
            bulk_g2s(st + SUB, page + MOFF, 16, &full[s]);
          }
        } else {
          const uint16_t *ks, *vs;
          uint32_t bytes;
          fp16_src(c, ug, sg.u, -tl - 1, R, k_new, v_new, ks, vs, bytes);
          mbar_arrive_expect_tx(&full[s], 2 * bytes);
          bulk_g2s(st, ks, bytes, &full[s]);
          bulk_g2s(st + OFF_FV, vs, bytes, &full[s]);
        }
      }
      (void)srow0;
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- consumers
    for (int si = 0; si < nseg; ++si) {
      const Seg sg = plan.seg[si];
      const int u = sg.u, b = u / c.Hkv, kvh = u % c.Hkv;
      int32_t* srow = state_row(c, b);
      const UnitGeo ug = geo_of_unit(c, u, R);
      uint32_t qf[8][2];
      load_q<KB>(c, q, b, kvh, G, g, t, qf);
      WarpState ws;
      ws.m[0] = ws.m[1] = -INFINITY;
      ws.l[0] = ws.l[1] = 0.f;
#pragma unroll
      for (int m = 0; m < 8; ++m) ws.o[m][0] = ws.o[m][1] = ws.o[m][2] = ws.o[m][3] = 0.f;
      // this warp's tiles of the segment: i = sg.a + ((warp - sg.a) mod NC), step NC
      int i = sg.a + ((warp - sg.a) % NC + NC) % NC;
      int held = -1;
      for (; i < sg.b; i += NC) {
        const int s = i % NSTAGES;
        // the timeout decision is made warp-uniform so the warp never splits
        if (!__all_sync(0xffffffffu, *reinterpret_cast<volatile int*>(&s_timeout) == 0 &&
                                         mbar_wait(&full[s], (i / NSTAGES) & 1, srow))) {
          if (lane == 0) s_timeout = 1;
          break;
        }
        const uint8_t* st = smem + s * STAGE_BYTES;
        const int tl = seg_tile(sg, i);
        if (tl >= 0) {
          packed_tile<KB, VB>(ws, st, qf, tl, ug.n_packed, qscale, g, t);
        } else {
          fp16_tile<KB>(ws, st, qf, fp16_valid(ug, -tl - 1, R), qscale, g, t);
        }
        __syncwarp();
        if (i + NC < sg.b) {
          if (lane == 0) mbar_arrive(&empty[s]);
        } else {
          held = s;  // the last tile of the segment: keep the stage for the warp state
        }
      }
      // l: sum the per-thread partial sums over the 8 lanes of a query column
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        ws.l[0] += __shfl_xor_sync(0xffffffffu, ws.l[0], o);
        ws.l[1] += __shfl_xor_sync(0xffffffffu, ws.l[1], o);
      }
      if (held >= 0) {
        float* wsm = reinterpret_cast<float*>(smem + held * STAGE_BYTES);
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
      if (lane == 0) s_held[warp] = held;
      segment_epilogue(c, q, k_new, v_new, out, parts, tickets, lse_ok, smem, s_held, &s_last, &s_glast, sg, ug, si, nseg);
      if (held >= 0 && lane == 0) mbar_arrive(&empty[held]);
    }
  }
  __syncthreads();  // every tile consumed
  if (s_timeout) {
    // never expected: before the CTA exits, wait (bounded) for every bulk copy
    // this CTA issued to land
    if (threadIdx.x == 0)
      for (int st = 0; st < NSTAGES; ++st)
        if (s_issued[st] > 0) mbar_wait(&full[st], (s_issued[st] - 1) & 1, state_row(c, 0));
    __syncthreads();
  }
}

}  // namespace

// counters: [0] grid ticket, [1 + u] unit tickets; zero between calls
size_t decode_counter_bytes(const hq_cache& c) { return ((4ull * (1 + c.B * c.Hkv) + 255) / 256) * 256; }

// partial slots: (CTA c, unit u) -> c + u, at most sms + units - 1 of them
size_t decode_workspace(const hq_cache& c, int sms) {
  return decode_counter_bytes(c) + (static_cast<size_t>(sms) + static_cast<size_t>(c.B) * c.Hkv) * PART_FLOATS * sizeof(float);
}

bool decode_supported(const hq_cache& c) {
  const int kb = kbits_of(c), vb = vbits_of(c);
  const bool fmt = (kb == 4 && vb == 4) || (kb == 8 && vb == 8) || (kb == 4 && vb == 2) || (kb == 2 && vb == 4);
  return fmt && c.B * c.Hkv <= MAX_UNITS;
}


hq_status launch_decode(const hq_cache& c, const uint16_t* q, const uint16_t* kn, const uint16_t* vn, uint16_t* out,
                        float sm_scale, void* ws, int sms, cudaStream_t st) {
  if (!decode_supported(c)) return HQ_ERR_UNSUPPORTED;
  const int smem = NSTAGES * STAGE_BYTES;
  int dev = 0;
  cudaGetDevice(&dev);
  static DeviceOnce attrs;
  const cudaError_t ea = attrs.run(dev, [] {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<4, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, NSTAGES * STAGE_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_kernel<8, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, NSTAGES * STAGE_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_kernel<4, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, NSTAGES * STAGE_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_kernel<2, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, NSTAGES * STAGE_BYTES);
    return e;
  });
  if (ea != cudaSuccess) return cuda_fail(ea, "decode attributes");
  unsigned int* tickets = reinterpret_cast<unsigned int*>(ws);
  float* parts = reinterpret_cast<float*>(static_cast<char*>(ws) + decode_counter_bytes(c));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(min(sms, MAX_CTAS), 1, 1);
  cfg.blockDim = dim3(NTHREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float qs = sm_scale * LOG2E;
  // the stored log-sum-exps serve the reselection only at its own scale 1/sqrt(D)
  const int lse_ok = sm_scale == 1.0f / sqrtf(static_cast<float>(D));
  const int kb = kbits_of(c), vb = vbits_of(c);
  cudaError_t e;
  if (kb == 8) e = cudaLaunchKernelEx(&cfg, decode_kernel<8, 8>, c, q, kn, vn, out, qs, parts, tickets, lse_ok);
  else if (vb == 2) e = cudaLaunchKernelEx(&cfg, decode_kernel<4, 2>, c, q, kn, vn, out, qs, parts, tickets, lse_ok);
  else if (kb == 2) e = cudaLaunchKernelEx(&cfg, decode_kernel<2, 4>, c, q, kn, vn, out, qs, parts, tickets, lse_ok);
  else e = cudaLaunchKernelEx(&cfg, decode_kernel<4, 4>, c, q, kn, vn, out, qs, parts, tickets, lse_ok);
  return cuda_status(e, "decode launch");
}

}  // namespace hq
