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
//   pack_rows      positions [lo, hi) of every (b, kv head) -> packed records
//   ring_fill      init only: last min(W, L) prefix rows -> FP16 ring
//   vl_gather      merge only: new VL rows -> workspace (old VL row, found through
//                  its page's bitmap, ring row, or the dequantised record rounded
//                  once to fp16)
//   vl_clear       merge only: bitmap words of the pages holding the old lines -> 0
//   vl_install     rows -> VL store, positions, bitmap bits, per-page first VL row,
//                  state update
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

// Rows [lo, hi) of every (b, kv head), K and V.  Init: src = dense [B,Hkv,L,D],
// lo = 0, hi = max(L - W, 0) for every sequence.  Merge: src = ring, and per
// sequence lo = n_packed, hi = T - W (from its state row; at most R rows, the
// ring's length, since the ring holds every position in [n_packed, T)).
__global__ void pack_rows_kernel(hq_cache c, const uint16_t* __restrict__ kd, const uint16_t* __restrict__ vd, int L,
                                 int init) {
  const Dims d = dims_of(c);
  const int nmax = init ? max(L - d.W, 0) : d.R;
  if (nmax <= 0) return;
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long total = 2ll * d.B * d.Hkv * nmax;  // (K or V) x (b, h) x rows
  for (long long w = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total; w += warps) {
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
      if (p >= hi) continue;
      src = (which ? c.vr : c.kr) + (bh * d.R + (p % d.R)) * D;
    }
    uint8_t* page = page_for_write(c, bh, p);
    if (page == nullptr) continue;
    const PageGeo pg = page_geo(c);
    pack_row_warp(src, row_codes(pg, page, which, p), row_sz(pg, page, which, p), lane, which ? pg.vb : pg.kb);
  }
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

// Merge: gather the FP16 rows of the new VL set into the workspace.  One warp
// per (b, h, row) handles K and V; an old line is found through its page's
// bitmap (read only here: the bits change in the next two kernels).
__global__ void vl_gather_kernel(hq_cache c, uint16_t* __restrict__ wsk, uint16_t* __restrict__ wsv) {
  const Dims d = dims_of(c);
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long total = static_cast<long long>(d.B) * d.Hkv * d.vl_cap;
  for (long long w = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total; w += warps) {
    const int r = static_cast<int>(w % d.vl_cap);
    const long long bh = w / d.vl_cap;
    int32_t* st = state_row(c, static_cast<int>(bh / d.Hkv));
    const int k = min(st[HQ_STATE_KSEL], d.vl_cap);
    if (r >= k) continue;
    const int n_packed = st[HQ_STATE_NPACKED];
    const int p = c.vl_sel[bh * d.vl_cap + r];
    if (p < 0 || p >= max(n_packed, st[HQ_STATE_T] - d.W)) {  // not a position the merge can hold
      if (lane == 0) set_err(st, HQ_DEVERR_VL_CAPACITY);
      continue;
    }
    const int old = p < n_packed ? old_vl_row(c, bh, p) : -1;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      uint16_t* dst = (which ? wsv : wsk) + (bh * d.vl_cap + r) * D;
      if (old >= 0) {
        const uint16_t* s = (which ? c.vf : c.kf) + (bh * d.vl_cap + old) * D;
        reinterpret_cast<uint2*>(dst)[lane] = reinterpret_cast<const uint2*>(s)[lane];
      } else if (p >= n_packed) {
        const uint16_t* s = (which ? c.vr : c.kr) + (bh * d.R + (p % d.R)) * D;
        reinterpret_cast<uint2*>(dst)[lane] = reinterpret_cast<const uint2*>(s)[lane];
      } else {
        // promoted packed position: fp16(zero + q * scale); q * scale is exact in
        // float64 and the sum is rounded once, then once more to fp16 (RN).
        // Lane l dequantises values 4l .. 4l+3 (4 * bits code bits).
        const PageGeo pg = page_geo(c);
        uint8_t* page = page_of(c, bh, p);
        const int bits = which ? pg.vb : pg.kb;
        const uint8_t* codes = row_codes(pg, page, which, p);
        const uint32_t szw = row_sz(pg, page, which, p)[lane >> 3];
        const double sc = static_cast<double>(__half2float(__ushort_as_half(static_cast<unsigned short>(szw & 0xFFFFu))));
        const double ze = static_cast<double>(__half2float(__ushort_as_half(static_cast<unsigned short>(szw >> 16))));
        const uint32_t qw = bits == 4 ? reinterpret_cast<const uint16_t*>(codes)[lane]
                                      : (bits == 8 ? reinterpret_cast<const uint32_t*>(codes)[lane] : codes[lane]);
        const uint32_t mask = (1u << bits) - 1u;
        uint32_t out[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const double v0 = __dadd_rn(ze, __dmul_rn(static_cast<double>((qw >> (bits * 2 * i)) & mask), sc));
          const double v1 = __dadd_rn(ze, __dmul_rn(static_cast<double>((qw >> (bits * (2 * i + 1))) & mask), sc));
          out[i] = static_cast<uint32_t>(__half_as_ushort(__double2half(v0))) |
                   (static_cast<uint32_t>(__half_as_ushort(__double2half(v1))) << 16);
        }
        reinterpret_cast<uint2*>(dst)[lane] = make_uint2(out[0], out[1]);
      }
    }
  }
}

// Merge: clear the bitmap words of every page that holds a current (old)
// vertical line (plain stores of zero; the new set's bits are set afterwards).
__global__ void vl_clear_kernel(hq_cache c) {
  const Dims d = dims_of(c);
  const long long total = static_cast<long long>(d.B) * d.Hkv * d.vl_cap;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long bh = i / d.vl_cap;
    const int r = static_cast<int>(i % d.vl_cap);
    if (r >= state_row(c, static_cast<int>(bh / d.Hkv))[HQ_STATE_NVL]) continue;
    uint8_t* page = page_for_write(c, bh, c.vl_pos[bh * d.vl_cap + r]);
    if (page) *reinterpret_cast<uint2*>(page_mask(page_geo(c), page)) = make_uint2(0u, 0u);
  }
}

// Install rows into the VL store.  Init: rows from the dense prefix; merge: rows
// from the workspace.  One warp per (b, h, row): K and V rows, vl_pos, the
// bitmap bit and (first line of a page) the page's first VL-store row.  The
// last block to finish (ticket) updates the state rows.
__global__ void vl_install_kernel(hq_cache c, const uint16_t* __restrict__ srck, const uint16_t* __restrict__ srcv, int L,
                                  int init, unsigned int* __restrict__ ticket) {
  const Dims d = dims_of(c);
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long total = static_cast<long long>(d.B) * d.Hkv * d.vl_cap;
  for (long long w = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total; w += warps) {
    const int row = static_cast<int>(w % d.vl_cap);
    const long long bh = w / d.vl_cap;
    int32_t* st = state_row(c, static_cast<int>(bh / d.Hkv));
    const int k = min(st[HQ_STATE_KSEL], d.vl_cap);
    if (row >= k) continue;
    const int p = c.vl_sel[bh * d.vl_cap + row];
    const int limit = init ? max(L - d.W, 0) : max(st[HQ_STATE_NPACKED], st[HQ_STATE_T] - d.W);
    if (p < 0 || p >= limit) {
      if (lane == 0) set_err(st, HQ_DEVERR_VL_CAPACITY);
      continue;
    }
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const uint16_t* s = init ? ((which ? srcv : srck) + (bh * L + p) * D)
                               : ((which ? srcv : srck) + (bh * d.vl_cap + row) * D);
      uint16_t* t = (which ? c.vf : c.kf) + (bh * d.vl_cap + row) * D;
      reinterpret_cast<uint2*>(t)[lane] = reinterpret_cast<const uint2*>(s)[lane];
    }
    if (lane == 0) {
      c.vl_pos[bh * d.vl_cap + row] = p;
      uint8_t* page = page_for_write(c, bh, p);
      if (page) {
        const PageGeo pg = page_geo(c);
        atomicOr(page_mask(pg, page) + ((p & 63) >> 5), 1u << (p & 31));
        // the first vertical line of a page records its VL-store row (rows are in
        // ascending position order), so readers find a line's row by a popcount
        if (row == 0 || (c.vl_sel[bh * d.vl_cap + row - 1] >> 6) != (p >> 6)) *page_vlbase(pg, page) = row;
      }
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
  if (init) clear_bitmaps_kernel<<<sms, threads, 0, st>>>(c);
  pack_rows_kernel<<<sms * 4, threads, 0, st>>>(c, kd, vd, L, init);
  if (init) {
    ring_fill_kernel<<<sms, threads, 0, st>>>(c, kd, vd, L);
    vl_install_kernel<<<sms * 4, threads, 0, st>>>(c, kd, vd, L, 1, ticket);
  } else {
    vl_gather_kernel<<<sms * 4, threads, 0, st>>>(c, wsk, wsv);
    vl_clear_kernel<<<sms, threads, 0, st>>>(c);
    vl_install_kernel<<<sms * 4, threads, 0, st>>>(c, wsk, wsv, L, 0, ticket);
  }
  return cuda_status(cudaGetLastError(), "merge launch");
}

hq_status launch_clear_bitmaps(const hq_cache& c, int sms, cudaStream_t st) {
  clear_bitmaps_kernel<<<sms, 256, 0, st>>>(c);
  return cuda_status(cudaGetLastError(), "reset bitmaps");
}

}  // namespace hq
