// pack_merge.cu — K4V4 packing and the staging -> hybrid merge.
//
// HyQuant digest (agihunt.info), prefill/decode paragraph: new decode tokens
// are staged first and merged into the hybrid layout later; the VL set chosen
// by the selector keeps FP16 rows, everything that leaves the recent window
// is stored 4-bit (or, with the cache's k_bits / v_bits, 2- or 8-bit; README
// Mode reference).  The arithmetic follows the format definition in hq.h
// exactly (float32 RN subtract/divide, rint to even, fp16 RN), so the packed
// bytes are bit-identical to the definition.
//
// Kernels (all bandwidth-trivial next to decode; one warp per row):
//   pack_rows      init only: prefix positions [0, L - W) of every (b, kv head)
//                  -> packed records
//   ring_fill      init only: last min(W, L) prefix rows -> FP16 ring
//   merge_gather   merge only, one launch for three kinds of item: the rows
//                  leaving the window -> packed records; new VL rows ->
//                  workspace (old VL row, found through its page's bitmap, ring
//                  row, or the dequantised record rounded once to fp16); the
//                  bitmap words of the pages that keep no line -> 0
//   vl_install     rows -> VL store, positions, each page's bitmap word and
//                  first VL row (written whole by the page's first line), state
//                  update
#include "common.cuh"

namespace hq {
namespace {

struct Dims {
  int B, Hkv, cap, vl_cap, R, W;
};

__device__ __forceinline__ Dims dims_of(const hq_cache& c) { return Dims{c.B, c.Hkv, c.cap, c.vl_cap, ring_len(c.W), c.W}; }

// Pack one 128-value fp16 row into 16 * bits code bytes + 4 (scale, zero)
// words, with 2^bits - 1 levels.  Warp-cooperative: lane l owns values 4l ..
// 4l+3 (group l / 8), i.e. 4 * bits consecutive bits of the codes.
__device__ __forceinline__ void pack_row_warp(const uint16_t* __restrict__ src, uint8_t* __restrict__ codes,
                                              uint32_t* __restrict__ sz, int lane, int bits) {
  const uint2 raw = *reinterpret_cast<const uint2*>(src + 4 * lane);
  float x[4];
  x[0] = __half2float(__ushort_as_half(static_cast<unsigned short>(raw.x & 0xFFFFu)));
  x[1] = __half2float(__ushort_as_half(static_cast<unsigned short>(raw.x >> 16)));
  x[2] = __half2float(__ushort_as_half(static_cast<unsigned short>(raw.y & 0xFFFFu)));
  x[3] = __half2float(__ushort_as_half(static_cast<unsigned short>(raw.y >> 16)));
  float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
  float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float levels = static_cast<float>((1 << bits) - 1);
  // scale = fp16_RN(fp32(mx - mn) / levels), zero = mn (an fp16 value, exact in fp32)
  const float span = __fsub_rn(mx, mn);
  const __half scale_h = __float2half_rn(__fdiv_rn(span, levels));
  const float scale = __half2float(scale_h);
  uint32_t q = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float r = scale == 0.0f ? 0.0f : rintf(__fdiv_rn(__fsub_rn(x[i], mn), scale));
    r = fminf(fmaxf(r, 0.0f), levels);
    q |= static_cast<uint32_t>(r) << (bits * i);
  }
  if (bits == 4) reinterpret_cast<uint16_t*>(codes)[lane] = static_cast<uint16_t>(q);
  else if (bits == 8) reinterpret_cast<uint32_t*>(codes)[lane] = q;
  else codes[lane] = static_cast<uint8_t>(q);
  if ((lane & 7) == 0) {
    const uint32_t zbits = __half_as_ushort(__float2half_rn(mn));  // exact: mn is an fp16 value
    sz[lane >> 3] = static_cast<uint32_t>(__half_as_ushort(scale_h)) | (zbits << 16);
  }
}

// Pack item w of 2 B Hkv nmax (K or V) x (b, h) x rows.  Init: src = dense
// [B,Hkv,L,D], rows [0, max(L - W, 0)) of every sequence.  Merge: src = ring,
// and per sequence rows [n_packed, T - W) (from its state row; at most R rows,
// the ring's length, since the ring holds every position in [n_packed, T)).
__device__ __forceinline__ void pack_item(const hq_cache& c, const Dims& d, const uint16_t* __restrict__ kd,
                                          const uint16_t* __restrict__ vd, int L, int init, int nmax, long long w,
                                          int lane) {
  const int which = static_cast<int>(w & 1);
  const long long rest = w >> 1;
  const int r = static_cast<int>(rest % nmax);
  const long long bh = rest / nmax;
  int p;
  const uint16_t* src;
  if (init) {
    p = r;
    src = (which ? vd : kd) + (bh * L + p) * D;
  } else {
    const int32_t* st = state_row(c, static_cast<int>(bh / d.Hkv));
    const int lo = st[HQ_STATE_NPACKED];
    const int hi = max(lo, st[HQ_STATE_T] - d.W);
    p = lo + r;
    if (p >= hi) return;
    src = (which ? c.vr : c.kr) + (bh * d.R + (p % d.R)) * D;
  }
  uint8_t* page = page_for_write(c, bh, p);
  if (page == nullptr) return;
  const PageGeo pg = page_geo(c);
  pack_row_warp(src, row_codes(pg, page, which, p), row_sz(pg, page, which, p), lane, which ? pg.vb : pg.kb);
}

// Init: the prefix rows [0, L - W) of every (b, kv head), K and V.
__global__ void pack_rows_kernel(hq_cache c, const uint16_t* __restrict__ kd, const uint16_t* __restrict__ vd, int L) {
  const Dims d = dims_of(c);
  const int nmax = max(L - d.W, 0);
  if (nmax <= 0) return;
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long total = 2ll * d.B * d.Hkv * nmax;
  for (long long w = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total; w += warps)
    pack_item(c, d, kd, vd, L, 1, nmax, w, lane);
}

// Init: prefix rows [max(L-W,0), L) -> ring slots p % R.
__global__ void ring_fill_kernel(hq_cache c, const uint16_t* __restrict__ kd, const uint16_t* __restrict__ vd, int L) {
  const Dims d = dims_of(c);
  const int lo = max(L - d.W, 0);
  const int n = L - lo;
  if (n <= 0) return;
  const long long total = 2ll * d.B * d.Hkv * n * (D / 8);  // 16-byte chunks
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int chunk = static_cast<int>(i % (D / 8));
    long long r = i / (D / 8);
    const int which = static_cast<int>(r & 1);
    r >>= 1;
    const int p = lo + static_cast<int>(r % n);
    const long long bh = r / n;
    const uint4* s = reinterpret_cast<const uint4*>((which ? vd : kd) + (bh * L + p) * D) + chunk;
    uint4* t = reinterpret_cast<uint4*>((which ? c.vr : c.kr) + (bh * d.R + (p % d.R)) * D) + chunk;
    *t = *s;
  }
}

// VL-store row of position p if p is one of the current vertical lines (its
// page's bitmap bit is set), else -1: the page records the row of its first
// line, and rows are in position order, so the row is that plus the number of
// lines of the page below p.
__device__ __forceinline__ int old_vl_row(const hq_cache& c, size_t bh, int p) {
  const PageGeo pg = page_geo(c);
  uint8_t* page = page_of(c, bh, p);
  const uint2 m = *reinterpret_cast<const uint2*>(page_mask(pg, page));
  const int r = p & 63;
  const uint32_t w = r < 32 ? m.x : m.y;
  if (!((w >> (r & 31)) & 1u)) return -1;
  const int below = __popc(w & ((1u << (r & 31)) - 1u)) + (r < 32 ? 0 : __popc(m.x));
  return *page_vlbase(pg, page) + below;
}

// Values 16 s .. 16 s + 15 of a packed row (codes: the row's 16 * BITS code
// bytes, value j at bit BITS * j; szw: the (scale, zero) word of their group)
// as fp16(zero + q * scale): q * scale is exact in float64 and the sum is
// rounded once, then once more to fp16 (RN).
template <int BITS>
__device__ __forceinline__ void dequant16(const uint8_t* __restrict__ codes, uint32_t szw, int s, uint4& o0, uint4& o1) {
  constexpr int NW = BITS / 2;  // 32-bit code words holding 16 values
  uint32_t cw[NW];
  if constexpr (BITS == 8) {
    const uint4 t = *reinterpret_cast<const uint4*>(codes + 16 * s);
    cw[0] = t.x;
    cw[1] = t.y;
    cw[2] = t.z;
    cw[3] = t.w;
  } else if constexpr (BITS == 4) {
    const uint2 t = *reinterpret_cast<const uint2*>(codes + 8 * s);
    cw[0] = t.x;
    cw[1] = t.y;
  } else {
    cw[0] = *reinterpret_cast<const uint32_t*>(codes + 4 * s);
  }
  const double sc = static_cast<double>(__half2float(__ushort_as_half(static_cast<unsigned short>(szw & 0xFFFFu))));
  const double ze = static_cast<double>(__half2float(__ushort_as_half(static_cast<unsigned short>(szw >> 16))));
  constexpr uint32_t mask = (1u << BITS) - 1u;
  uint32_t h[8];
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const uint32_t q0 = (cw[(BITS * i) >> 5] >> ((BITS * i) & 31)) & mask;
    const uint32_t q1 = (cw[(BITS * (i + 1)) >> 5] >> ((BITS * (i + 1)) & 31)) & mask;
    const double v0 = __dadd_rn(ze, __dmul_rn(static_cast<double>(q0), sc));
    const double v1 = __dadd_rn(ze, __dmul_rn(static_cast<double>(q1), sc));
    h[i / 2] = static_cast<uint32_t>(__half_as_ushort(__double2half(v0))) |
               (static_cast<uint32_t>(__half_as_ushort(__double2half(v1))) << 16);
  }
  o0 = make_uint4(h[0], h[1], h[2], h[3]);
  o1 = make_uint4(h[4], h[5], h[6], h[7]);
}

// Does the new VL set hold a line of page pg (positions 64 pg .. 64 pg + 63)
// that the merge installs (below limit)?  The set is in ascending position
// order: a binary search for its first position at or above 64 pg.
__device__ __forceinline__ bool new_line_in_page(const int32_t* __restrict__ sel, int k, int pg, int limit) {
  int lo = 0, hi = k;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (sel[mid] < pg * HQ_PAGE_POSITIONS) lo = mid + 1;
    else hi = mid;
  }
  return lo < k && sel[lo] < min((pg + 1) * HQ_PAGE_POSITIONS, limit);
}

// Merge, first launch.  One index space of warp items, in three kinds:
//   [0, n_pack)                   pack one row leaving the window (K or V);
//   [n_pack, + B Hkv ceil(vl_cap/4)) gather 4 rows of the new VL set into the
//                                 workspace, 8 lanes per row, K and V; an old
//                                 line is found through its page's bitmap;
//   [.., + B Hkv ceil(vl_cap/32)) 32 rows of the old VL set: the bitmap words
//                                 of the pages where the new set keeps no line
//                                 -> 0 (the install writes the others whole).
// No item reads what another writes: packing writes the records of positions
// at or above n_packed, which no gather reads; a gather reads the bitmap of a
// page that holds a new line, and only pages without one are zeroed.
__global__ void merge_gather_kernel(hq_cache c, uint16_t* __restrict__ wsk, uint16_t* __restrict__ wsv) {
  const Dims d = dims_of(c);
  const int lane = threadIdx.x & 31;
  const long long nbh = static_cast<long long>(d.B) * d.Hkv;
  const long long n_pack = 2ll * nbh * d.R;
  const int rq = (d.vl_cap + 3) / 4;
  const long long n_gather = nbh * rq;
  const int cw = (d.vl_cap + 31) / 32;
  const long long total = n_pack + n_gather + nbh * cw;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long w = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total; w += warps) {
    if (w < n_pack) {
      pack_item(c, d, nullptr, nullptr, 0, 0, d.R, w, lane);
      continue;
    }
    if (w >= n_pack + n_gather) {
      const long long i = w - n_pack - n_gather;
      const long long bh = i / cw;
      const int r = static_cast<int>(i % cw) * 32 + lane;
      const int32_t* st = state_row(c, static_cast<int>(bh / d.Hkv));
      if (r >= st[HQ_STATE_NVL]) continue;
      const int32_t* pos = c.vl_pos + bh * d.vl_cap;
      const int p = pos[r];
      // the old set is in ascending position order too: one lane per page
      if (p < 0 || (r > 0 && (pos[r - 1] >> 6) == (p >> 6))) continue;
      const int k = min(st[HQ_STATE_KSEL], d.vl_cap);
      const int limit = max(st[HQ_STATE_NPACKED], st[HQ_STATE_T] - d.W);
      if (new_line_in_page(c.vl_sel + bh * d.vl_cap, k, p >> 6, limit)) continue;
      uint8_t* page = page_for_write(c, bh, p);
      if (page) *reinterpret_cast<uint2*>(page_mask(page_geo(c), page)) = make_uint2(0u, 0u);
      continue;
    }
    const long long g = w - n_pack;
    const int sub = lane & 7;  // 16 of the row's 128 values: 2 x 16 bytes of fp16
    const int r = static_cast<int>(g % rq) * 4 + (lane >> 3);
    const long long bh = g / rq;
    int32_t* st = state_row(c, static_cast<int>(bh / d.Hkv));
    const int k = min(st[HQ_STATE_KSEL], d.vl_cap);
    if (r >= k) continue;
    const int n_packed = st[HQ_STATE_NPACKED];
    const int p = c.vl_sel[bh * d.vl_cap + r];
    if (p < 0 || p >= max(n_packed, st[HQ_STATE_T] - d.W)) {  // not a position the merge can hold
      if (sub == 0) set_err(st, HQ_DEVERR_VL_CAPACITY);
      continue;
    }
    const int old = p < n_packed ? old_vl_row(c, bh, p) : -1;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      uint4* dst = reinterpret_cast<uint4*>((which ? wsv : wsk) + (bh * d.vl_cap + r) * D) + 2 * sub;
      if (old >= 0 || p >= n_packed) {
        const uint16_t* src = old >= 0 ? (which ? c.vf : c.kf) + (bh * d.vl_cap + old) * D
                                       : (which ? c.vr : c.kr) + (bh * d.R + (p % d.R)) * D;
        const uint4* s4 = reinterpret_cast<const uint4*>(src) + 2 * sub;
        const uint4 x0 = s4[0], x1 = s4[1];
        dst[0] = x0;
        dst[1] = x1;
      } else {
        // promoted packed position: the record dequantised once
        const PageGeo pg = page_geo(c);
        uint8_t* page = page_of(c, bh, p);
        const int bits = which ? pg.vb : pg.kb;
        const uint8_t* codes = row_codes(pg, page, which, p);
        const uint32_t szw = row_sz(pg, page, which, p)[sub >> 1];
        uint4 o0, o1;
        if (bits == 4) dequant16<4>(codes, szw, sub, o0, o1);
        else if (bits == 8) dequant16<8>(codes, szw, sub, o0, o1);
        else dequant16<2>(codes, szw, sub, o0, o1);
        dst[0] = o0;
        dst[1] = o1;
      }
    }
  }
}

// Install rows into the VL store.  Init: rows from the dense prefix; merge: rows
// from the workspace.  One warp per 4 rows of a (b, h), 8 lanes per row: K and
// V rows and vl_pos; the first line of a page writes the page's bitmap word
// whole (every line of the set in that page: they follow it in position order)
// and its first VL-store row.  The last block to finish (ticket) updates the
// state rows.
__global__ void vl_install_kernel(hq_cache c, const uint16_t* __restrict__ srck, const uint16_t* __restrict__ srcv, int L,
                                  int init, unsigned int* __restrict__ ticket) {
  const Dims d = dims_of(c);
  const int lane = threadIdx.x & 31;
  const int sub = lane & 7;                            // 16 of the row's 128 values
  const unsigned int gmask = 0xFFu << (lane & ~7);     // the row's 8 lanes
  const int rq = (d.vl_cap + 3) / 4;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long total = static_cast<long long>(d.B) * d.Hkv * rq;
  for (long long w = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total; w += warps) {
    const int row = static_cast<int>(w % rq) * 4 + (lane >> 3);
    const long long bh = w / rq;
    int32_t* st = state_row(c, static_cast<int>(bh / d.Hkv));
    const int k = min(st[HQ_STATE_KSEL], d.vl_cap);
    if (row >= k) continue;  // the same for the row's 8 lanes, as is every branch below
    const int32_t* sel = c.vl_sel + bh * d.vl_cap;
    const int p = sel[row];
    const int limit = init ? max(L - d.W, 0) : max(st[HQ_STATE_NPACKED], st[HQ_STATE_T] - d.W);
    if (p < 0 || p >= limit) {
      if (sub == 0) set_err(st, HQ_DEVERR_VL_CAPACITY);
      continue;
    }
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const uint16_t* src = init ? ((which ? srcv : srck) + (bh * L + p) * D)
                                 : ((which ? srcv : srck) + (bh * d.vl_cap + row) * D);
      const uint4* s4 = reinterpret_cast<const uint4*>(src) + 2 * sub;
      uint4* t4 = reinterpret_cast<uint4*>((which ? c.vf : c.kf) + (bh * d.vl_cap + row) * D) + 2 * sub;
      const uint4 x0 = s4[0], x1 = s4[1];
      t4[0] = x0;
      t4[1] = x1;
    }
    if (sub == 0) c.vl_pos[bh * d.vl_cap + row] = p;
    if (row > 0 && (sel[row - 1] >> 6) == (p >> 6)) continue;
    // the first vertical line of its page: the page's bitmap word, and its
    // VL-store row (rows are in ascending position order), so readers find a
    // line's row by a popcount.  The page's lines are the rows from here on
    // while they stay in the page: 8 of them per round, one per lane.
    const long long idx = page_index(c, bh, p >> 6);
    if (idx < 0) {
      if (sub == 0) set_err(st, HQ_DEVERR_PAGE);
      continue;
    }
    uint32_t m0 = 0u, m1 = 0u;
    for (int j0 = row; j0 < k; j0 += 8) {
      const int j = j0 + sub;
      const int pj = j < k ? sel[j] : -1;
      const bool in = j < k && (pj >> 6) == (p >> 6) && pj < limit;
      if (in) {
        if (pj & 32) m1 |= 1u << (pj & 31);
        else m0 |= 1u << (pj & 31);
      }
      if (((__ballot_sync(gmask, in) >> (lane & ~7)) & 0xFFu) != 0xFFu) break;
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      m0 |= __shfl_xor_sync(gmask, m0, o);
      m1 |= __shfl_xor_sync(gmask, m1, o);
    }
    if (sub == 0) {
      const PageGeo pg = page_geo(c);
      uint8_t* page = c.pages + static_cast<size_t>(idx) * pg.bytes;
      *reinterpret_cast<uint2*>(page_mask(pg, page)) = make_uint2(m0, m1);
      *page_vlbase(pg, page) = row;
    }
  }
  // state update by the last block (every block has read the state rows above)
  __syncthreads();
  __shared__ unsigned int last;
  if (threadIdx.x == 0) {
    __threadfence();
    last = (atomicAdd(ticket, 1u) == gridDim.x - 1) ? 1u : 0u;
  }
  __syncthreads();
  if (last) {
    for (int b = threadIdx.x; b < d.B; b += blockDim.x) {
      int32_t* st = state_row(c, b);
      if (init) {
        st[HQ_STATE_T] = L;
        st[HQ_STATE_NPACKED] = max(L - d.W, 0);
        st[HQ_STATE_NQ] = 0;
      } else {
        st[HQ_STATE_NPACKED] = max(st[HQ_STATE_NPACKED], st[HQ_STATE_T] - d.W);
      }
      st[HQ_STATE_NVL] = min(st[HQ_STATE_KSEL], d.vl_cap);
    }
    if (threadIdx.x == 0) *ticket = 0u;
  }
}

// Clear the VL bitmap of every page the descriptor's sequences own (through
// the page table when there is one); entries outside the pool are skipped.
__global__ void clear_bitmaps_kernel(hq_cache c) {
  const int npg = c.cap / HQ_PAGE_POSITIONS;
  const long long total = static_cast<long long>(c.B) * c.Hkv * npg;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long idx = page_index(c, static_cast<size_t>(i / npg), static_cast<int>(i % npg));
    if (idx < 0) continue;
    const PageGeo pg = page_geo(c);
    *reinterpret_cast<uint2*>(c.pages + static_cast<size_t>(idx) * pg.bytes + pg.mask) = make_uint2(0u, 0u);
  }
}

}  // namespace

// ------------------------------------------------------------------ host launchers

hq_status launch_pack_merge(const hq_cache& c, const uint16_t* kd, const uint16_t* vd, int L, void* ws, cudaStream_t st) {
  const int init = kd != nullptr;
  const int threads = 256;
  int sms = 148;
  {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  unsigned int* ticket = reinterpret_cast<unsigned int*>(ws);
  uint16_t* wsk = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + 256);
  uint16_t* wsv = wsk + static_cast<size_t>(c.B) * c.Hkv * c.vl_cap * D;
  // warp items -> blocks of 8 warps, at most 8 blocks per SM (one wave)
  const auto blocks = [&](long long items) {
    return static_cast<int>(max(1ll, min((items + 7) / 8, 8ll * sms)));
  };
  const long long nbh = static_cast<long long>(c.B) * c.Hkv;
  const long long install_items = nbh * ((c.vl_cap + 3) / 4);
  if (init) {
    clear_bitmaps_kernel<<<sms, threads, 0, st>>>(c);
    pack_rows_kernel<<<sms * 4, threads, 0, st>>>(c, kd, vd, L);
    ring_fill_kernel<<<sms, threads, 0, st>>>(c, kd, vd, L);
    vl_install_kernel<<<blocks(install_items), threads, 0, st>>>(c, kd, vd, L, 1, ticket);
  } else {
    const long long gather_items = 2 * nbh * ring_len(c.W) + nbh * ((c.vl_cap + 3) / 4) + nbh * ((c.vl_cap + 31) / 32);
    merge_gather_kernel<<<blocks(gather_items), threads, 0, st>>>(c, wsk, wsv);
    vl_install_kernel<<<blocks(install_items), threads, 0, st>>>(c, wsk, wsv, L, 0, ticket);
  }
  return cuda_status(cudaGetLastError(), "merge launch");
}

hq_status launch_clear_bitmaps(const hq_cache& c, int sms, cudaStream_t st) {
  clear_bitmaps_kernel<<<sms, 256, 0, st>>>(c);
  return cuda_status(cudaGetLastError(), "reset bitmaps");
}

}  // namespace hq
