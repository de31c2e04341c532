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
// Kernels
//   select_pass<LSE>   per key chunk of 128: S = Q . K^T on tensor cores
//                      (mma.m16n8k16, keys rebuilt in shared memory in their
//                      current representation) -> per-(query, chunk) running
//                      max / sum in the exp2 domain
//   lse_merge          per-query log-sum-exp over the chunks
//   select_pass<COL>   recompute S, p = exp2(S - lse), column sums over all
//                      queries of the group -> score_j (no atomics in global
//                      memory: one CTA owns each key)
//   topk               one CTA per (b, kv head): 4 rounds of 8-bit radix
//                      select on the float bit patterns (scores are >= 0, so
//                      the bit order is the value order) -> exact k-th value,
//                      then a block scan writes the chosen positions in
//                      ascending order, ties to the lowest positions
#include "common.cuh"

namespace hq {
namespace {

constexpr int CH = 128;          // keys per chunk
constexpr int SROW = 272;        // bytes per fp16 row in shared memory
constexpr int NT_SEL = 256;      // threads
constexpr int NW_SEL = NT_SEL / 32;

struct SelArgs {
  hq_cache c;
  const uint16_t* k_dense;  // init mode: [B, Hkv, L, D]
  const uint16_t* q_ext;    // init mode: [B, Hq, nq, D]
  int L;                    // init mode length
  int nq_init;
  float* lse_part;          // [B*Hkv, C, M] x (m, l)
  float* lse;               // [B*Hkv, M]
  float* scores;            // [B*Hkv, cap]
  int C;                    // chunks in the grid (cap / CH)
  float qscale;             // sm_scale * log2(e)
};

struct SelGeo {
  int T, n, nq, qpos0, n_packed, n_vl;
};

__device__ __forceinline__ SelGeo sel_geo(const SelArgs& a) {
  SelGeo g;
  if (a.k_dense) {
    g.T = a.L;
    g.nq = a.nq_init;
    g.n_packed = 0;
    g.n_vl = 0;
  } else {
    g.T = a.c.state[HQ_STATE_T];
    g.nq = min(a.c.state[HQ_STATE_NQ], HQ_QBUF);
    g.n_packed = a.c.state[HQ_STATE_NPACKED];
    g.n_vl = a.c.state[HQ_STATE_NVL];
  }
  g.n = max(g.T - a.c.W, 0);
  g.qpos0 = g.T - g.nq;
  return g;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ int find_sorted(const int32_t* __restrict__ a, int n, int key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < key) lo = mid + 1; else hi = mid;
  }
  return (lo < n && a[lo] == key) ? lo : -1;
}

// Fill shared memory with keys [j0, j0 + CH) of (b, kv head) in their current
// representation (fp16).  One warp per key row; lane l owns dims 4l .. 4l+3.
__device__ void load_keys(const SelArgs& a, const SelGeo& g, int bh, int j0, uint8_t* ks) {
  const hq_cache& c = a.c;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int R = ring_len(c.W);
  for (int r = warp; r < CH; r += NW_SEL) {
    const int p = j0 + r;
    uint2 v = make_uint2(0u, 0u);
    if (p < g.T) {
      if (a.k_dense) {
        v = reinterpret_cast<const uint2*>(a.k_dense + (static_cast<size_t>(bh) * a.L + p) * D)[lane];
      } else if (p >= g.n_packed) {
        v = reinterpret_cast<const uint2*>(c.kr + (static_cast<size_t>(bh) * R + (p % R)) * D)[lane];
      } else if ((page_mask(page_of(c, bh, p))[(p & 63) >> 5] >> (p & 31)) & 1u) {
        const int idx = find_sorted(c.vl_pos + static_cast<size_t>(bh) * c.vl_cap, g.n_vl, p);
        if (idx >= 0) v = reinterpret_cast<const uint2*>(c.kf + (static_cast<size_t>(bh) * c.vl_cap + idx) * D)[lane];
      } else {
        uint8_t* page = page_of(c, bh, p);
        const uint32_t two = reinterpret_cast<const uint16_t*>(row_codes(page, 0, p))[lane];
        const uint32_t szw = row_sz(page, 0, p)[lane >> 3];
        const uint32_t s2 = prmt(szw, szw, 0x1010), z2 = prmt(szw, szw, 0x3232);
        // nibbles of byte 0 -> dims 4l, 4l+1 ; byte 1 -> dims 4l+2, 4l+3
        const uint32_t x0 = prmt(two, 0u, 0x4040);   // byte0 at bits 0..7 and 16..23
        const uint32_t x1 = prmt(two, 0u, 0x4141);   // byte1 at bits 0..7 and 16..23
        // low nibble -> .x, high nibble (bits 20..23) -> .y
        const uint32_t n0 = hfma2_u(and_or(x0, 0x00F0000Fu, MAGIC), 0x2C003C00u, 0xD400E400u);
        const uint32_t n1 = hfma2_u(and_or(x1, 0x00F0000Fu, MAGIC), 0x2C003C00u, 0xD400E400u);
        v.x = hfma2_u(n0, s2, z2);
        v.y = hfma2_u(n1, s2, z2);
      }
    }
    *reinterpret_cast<uint2*>(ks + r * SROW + 8 * lane) = v;
  }
}

template <bool COL>
__global__ void __launch_bounds__(NT_SEL) select_pass(SelArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const hq_cache& c = a.c;
  const int chunk = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int bh = b * c.Hkv + kvh;
  const int G = c.Hq / c.Hkv;
  const SelGeo g = sel_geo(a);
  const int M = G * g.nq;
  const int j0 = chunk * CH;
  const int lim = COL ? g.n : g.T;  // keys scored in this pass
  if (j0 >= lim || M == 0) return;

  uint8_t* qs = smem;
  uint8_t* ks = smem + static_cast<size_t>(M) * SROW;
  float* colsum = reinterpret_cast<float*>(ks + CH * SROW);   // [NW_SEL][CH], one row per warp
  float* lse_s = colsum + NW_SEL * CH;                          // [M]

  // queries: row r = h * nq + i  (head kvh*G + h, position qpos0 + i)
  for (int e = threadIdx.x; e < M * (D / 8); e += NT_SEL) {
    const int r = e / (D / 8), ch = e % (D / 8);
    const int h = r / g.nq, i = r % g.nq;
    const uint4* src;
    if (a.k_dense) {
      src = reinterpret_cast<const uint4*>(a.q_ext + ((static_cast<size_t>(b) * c.Hq + kvh * G + h) * g.nq + i) * D) + ch;
    } else {
      const int p = g.qpos0 + i;
      src = reinterpret_cast<const uint4*>(c.qbuf + ((static_cast<size_t>(b) * c.Hq + kvh * G + h) * HQ_QBUF + (p % HQ_QBUF)) * D) + ch;
    }
    *reinterpret_cast<uint4*>(qs + r * SROW + 16 * ch) = *src;
  }
  load_keys(a, g, bh, j0, ks);
  if (COL) {
    for (int i = threadIdx.x; i < NW_SEL * CH; i += NT_SEL) colsum[i] = 0.f;
    for (int i = threadIdx.x; i < M; i += NT_SEL) lse_s[i] = a.lse[static_cast<size_t>(bh) * (G * HQ_QBUF) + i];
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int nmt = (M + 15) / 16;
  for (int mt = warp; mt < nmt; mt += NW_SEL) {
    float acc[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a0, a1, a2, a3;
      {
        const int row = 16 * mt + (lane & 15);
        const int col = 16 * kk + 8 * (lane >> 4);
        ldsm_x4(smem_u32(qs + min(row, M - 1) * SROW + 2 * col), a0, a1, a2, a3);
      }
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        // keys 16np .. 16np+15: x4 = (keys 0-7, dims 0-7), (keys 0-7, dims 8-15), (keys 8-15, dims 0-7), (keys 8-15, dims 8-15)
        uint32_t b0, b1, b2, b3;
        const int key = 16 * np + (lane & 7) + 8 * (lane >> 4);
        const int col = 16 * kk + 8 * ((lane >> 3) & 1);
        ldsm_x4(smem_u32(ks + key * SROW + 2 * col), b0, b1, b2, b3);
        mma16816(acc[2 * np], a0, a1, a2, a3, b0, b1);
        mma16816(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    // rows of this thread: r0 = 16mt + gq, r1 = r0 + 8 ; keys 8n + 2tq + {0,1}
    const int r0 = 16 * mt + gq, r1 = r0 + 8;
    const int p0 = g.qpos0 + (r0 % max(g.nq, 1)), p1 = g.qpos0 + (r1 % max(g.nq, 1));
    const bool ok0 = r0 < M, ok1 = r1 < M;
    if (!COL) {
      float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = j0 + 8 * n + 2 * tq + e;
          if (j < lim && j <= p0) m0 = fmaxf(m0, acc[n][e] * a.qscale);
          if (j < lim && j <= p1) m1 = fmaxf(m1, acc[n][2 + e] * a.qscale);
        }
      }
      m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
      m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
      m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
      m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
      float l0 = 0.f, l1 = 0.f;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = j0 + 8 * n + 2 * tq + e;
          if (j < lim && j <= p0) l0 += ex2(acc[n][e] * a.qscale - m0);
          if (j < lim && j <= p1) l1 += ex2(acc[n][2 + e] * a.qscale - m1);
        }
      }
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      if (tq == 0) {
        float* lp = a.lse_part + (static_cast<size_t>(bh) * a.C + chunk) * (G * HQ_QBUF) * 2;
        if (ok0) { lp[2 * r0] = m0; lp[2 * r0 + 1] = l0; }
        if (ok1) { lp[2 * r1] = m1; lp[2 * r1 + 1] = l1; }
      }
    } else {
      const float z0 = ok0 ? lse_s[r0] : INFINITY, z1 = ok1 ? lse_s[r1] : INFINITY;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = j0 + 8 * n + 2 * tq + e;
          float v = 0.f;
          if (ok0 && j < lim && j <= p0) v += ex2(acc[n][e] * a.qscale - z0);
          if (ok1 && j < lim && j <= p1) v += ex2(acc[n][2 + e] * a.qscale - z1);
          // sum over the 8 row-groups of the warp (lanes with equal tq)
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          if (gq == 0) colsum[warp * CH + 8 * n + 2 * tq + e] += v;
        }
      }
    }
  }
  if (COL) {
    __syncthreads();
    for (int i = threadIdx.x; i < CH; i += NT_SEL) {
      const int j = j0 + i;
      if (j < lim) {
        float tot = 0.f;
        for (int w = 0; w < NW_SEL; ++w) tot += colsum[w * CH + i];  // fixed order: deterministic
        a.scores[static_cast<size_t>(bh) * c.cap + j] = tot;
      }
    }
  }
}

// lse (exp2 domain) per query row over the chunks that hold keys
__global__ void lse_merge(SelArgs a) {
  const hq_cache& c = a.c;
  const int bh = blockIdx.x;
  const int G = c.Hq / c.Hkv;
  const SelGeo g = sel_geo(a);
  const int M = G * g.nq;
  const int nch = (g.T + CH - 1) / CH;
  for (int r = threadIdx.x; r < M; r += blockDim.x) {
    float mm = -INFINITY;
    for (int ch = 0; ch < nch; ++ch) mm = fmaxf(mm, a.lse_part[((static_cast<size_t>(bh) * a.C + ch) * (G * HQ_QBUF)) * 2 + 2 * r]);
    float ll = 0.f;
    for (int ch = 0; ch < nch; ++ch) {
      const float* lp = a.lse_part + ((static_cast<size_t>(bh) * a.C + ch) * (G * HQ_QBUF)) * 2 + 2 * r;
      if (lp[0] != -INFINITY) ll += lp[1] * ex2(lp[0] - mm);
    }
    a.lse[static_cast<size_t>(bh) * (G * HQ_QBUF) + r] = mm + log2f(ll);
  }
}

constexpr int TK_THREADS = 1024;

// Exact top-k by radix select over the fp32 bit patterns (scores >= 0).
__global__ void __launch_bounds__(TK_THREADS) topk_kernel(SelArgs a) {
  const hq_cache& c = a.c;
  const int bh = blockIdx.x;
  const SelGeo g = sel_geo(a);
  const int n = g.n;
  int k = 0;
  if (n > 0 && c.rho_bp > 0) {
    const long long kk = (static_cast<long long>(n) * c.rho_bp + 9999) / 10000;
    k = static_cast<int>(min(static_cast<long long>(n), kk));
  }
  if (k > c.vl_cap) {
    if (bh == 0 && threadIdx.x == 0) set_err(c.state, HQ_DEVERR_VL_CAPACITY);
    k = c.vl_cap;
  }
  if (bh == 0 && threadIdx.x == 0) c.state[HQ_STATE_KSEL] = k;
  if (k == 0) return;
  const uint32_t* sc = reinterpret_cast<const uint32_t*>(a.scores + static_cast<size_t>(bh) * c.cap);
  int32_t* out = c.vl_sel + static_cast<size_t>(bh) * c.vl_cap;

  __shared__ unsigned int hist[256];
  __shared__ unsigned int s_prefix, s_need;
  __shared__ unsigned int warp_sums[TK_THREADS / 32][2];
  if (threadIdx.x == 0) {
    s_prefix = 0u;
    s_need = static_cast<unsigned>(k);
  }
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int i = threadIdx.x; i < 256; i += TK_THREADS) hist[i] = 0u;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    for (int j = threadIdx.x; j < n; j += TK_THREADS) {
      const uint32_t v = sc[j];
      if ((v & hi_mask) == (prefix & hi_mask)) atomicAdd(&hist[(v >> shift) & 0xFFu], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned int need = s_need, acc = 0u;
      int d = 255;
      for (; d > 0; --d) {
        if (acc + hist[d] >= need) break;
        acc += hist[d];
      }
      s_prefix = prefix | (static_cast<uint32_t>(d) << shift);
      s_need = need - acc;
    }
    __syncthreads();
  }
  const uint32_t thr = s_prefix;      // exact k-th largest value
  const unsigned int take_eq = s_need;  // how many values equal to thr to take (lowest positions first)

  // ordered compaction: each thread owns a contiguous segment
  const int per = (n + TK_THREADS - 1) / TK_THREADS;
  const int lo = threadIdx.x * per, hi = min(n, lo + per);
  unsigned int cnt_gt = 0, cnt_eq = 0;
  for (int j = lo; j < hi; ++j) {
    const uint32_t v = sc[j];
    cnt_gt += v > thr;
    cnt_eq += v == thr;
  }
  // block exclusive scan of (cnt_gt, cnt_eq)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned int x = cnt_gt, y = cnt_eq;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int xo = __shfl_up_sync(0xffffffffu, x, o), yo = __shfl_up_sync(0xffffffffu, y, o);
    if (lane >= o) { x += xo; y += yo; }
  }
  if (lane == 31) { warp_sums[warp][0] = x; warp_sums[warp][1] = y; }
  __syncthreads();
  if (warp == 0) {
    unsigned int wx = lane < TK_THREADS / 32 ? warp_sums[lane][0] : 0u;
    unsigned int wy = lane < TK_THREADS / 32 ? warp_sums[lane][1] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned int xo = __shfl_up_sync(0xffffffffu, wx, o), yo = __shfl_up_sync(0xffffffffu, wy, o);
      if (lane >= o) { wx += xo; wy += yo; }
    }
    if (lane < TK_THREADS / 32) { warp_sums[lane][0] = wx; warp_sums[lane][1] = wy; }
  }
  __syncthreads();
  unsigned int ex_gt = x - cnt_gt + (warp > 0 ? warp_sums[warp - 1][0] : 0u);
  unsigned int ex_eq = y - cnt_eq + (warp > 0 ? warp_sums[warp - 1][1] : 0u);
  // output slot of position j = (#gt before j) + min(#eq before j, take_eq)
  for (int j = lo; j < hi; ++j) {
    const uint32_t v = sc[j];
    if (v > thr) {
      out[ex_gt + min(ex_eq, take_eq)] = j;
      ++ex_gt;
    } else if (v == thr) {
      if (ex_eq < take_eq) out[ex_gt + ex_eq] = j;
      ++ex_eq;
    }
  }
}

}  // namespace

size_t select_smem_bytes(const hq_cache& c) {
  const int M = (c.Hq / c.Hkv) * HQ_QBUF;
  return static_cast<size_t>(M) * SROW + CH * SROW + NW_SEL * CH * 4 + M * 4;
}

size_t select_workspace(const hq_cache& c, bool need_scores) {
  const int M = (c.Hq / c.Hkv) * HQ_QBUF;
  const int C = c.cap / CH;
  size_t bytes = static_cast<size_t>(c.B) * c.Hkv * C * M * 2 * 4;  // lse partials
  bytes += static_cast<size_t>(c.B) * c.Hkv * M * 4;                  // lse
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
  const int M = (c.Hq / c.Hkv) * HQ_QBUF;
  // init mode: keys come from the dense prefix, which may be longer than cap
  const int keys_cap = kd ? ((L + CH - 1) / CH) * CH : c.cap;
  a.C = keys_cap / CH;
  char* w = static_cast<char*>(ws);
  a.lse_part = reinterpret_cast<float*>(w);
  w += static_cast<size_t>(c.B) * c.Hkv * a.C * M * 2 * 4;
  a.lse = reinterpret_cast<float*>(w);
  w += static_cast<size_t>(c.B) * c.Hkv * M * 4;
  a.scores = scores_out ? scores_out : reinterpret_cast<float*>(w);
  a.qscale = (1.0f / sqrtf(static_cast<float>(D))) * LOG2E;
  const size_t smem = select_smem_bytes(c);
  // the attribute is raised once per device to the size of the largest group (HQ_MAX_GQA)
  hq_cache cmax = c;
  cmax.Hq = cmax.Hkv * HQ_MAX_GQA;
  const int smem_max = static_cast<int>(select_smem_bytes(cmax));
  int dev = 0;
  cudaGetDevice(&dev);
  static bool attr_done[64] = {};
  if (dev >= 64 || !attr_done[dev]) {
    if (cudaFuncSetAttribute(select_pass<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max) != cudaSuccess ||
        cudaFuncSetAttribute(select_pass<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max) != cudaSuccess)
      return HQ_ERR_CUDA;
    if (dev < 64) attr_done[dev] = true;
  }
  dim3 grid(a.C, c.Hkv, c.B);
  select_pass<false><<<grid, NT_SEL, smem, st>>>(a);
  lse_merge<<<c.B * c.Hkv, 256, 0, st>>>(a);
  select_pass<true><<<grid, NT_SEL, smem, st>>>(a);
  topk_kernel<<<c.B * c.Hkv, TK_THREADS, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

}  // namespace hq
