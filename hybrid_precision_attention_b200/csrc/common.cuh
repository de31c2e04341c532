// common.cuh — small device helpers shared by the libhq kernels (sm_100a).
//
// Hand-written inline PTX for: mbarrier phases with bounded waits, 1-D bulk
// async copies (cp.async.bulk, non-multicast) into shared memory, legacy
// mma.sync tiles used by the bandwidth-bound decode scan, movmatrix, and the
// ex2 instruction.  No library math is reproduced here.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/hq.h"

namespace hq {

constexpr int D = HQ_HEAD_DIM;
constexpr float LOG2E = 1.4426950408889634f;

__host__ __device__ __forceinline__ int ring_len(int W) { return HQ_RING_LEN(W); }

// Host side: HQ_OK when e is cudaSuccess, else HQ_ERR_CUDA after recording the
// CUDA error name and `where` for hq_last_error() (per host thread).
hq_status cuda_status(cudaError_t e, const char* where);
// Host side: a failure path; always HQ_ERR_CUDA, recording `where` and e.
hq_status cuda_fail(cudaError_t e, const char* where);

// Host side: runs `set` (a kernel-attribute set-up) once per device for one
// call site.  Thread-safe: concurrent first calls on a device wait for the one
// that runs `set`; a failed set-up is not recorded, so the next call retries.
struct DeviceOnce {
  static constexpr int kMaxDevices = 64;
  std::atomic<bool> done[kMaxDevices] = {};
  std::mutex mu;
  template <class F>
  cudaError_t run(int dev, F&& set) {
    if (dev >= 0 && dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < kMaxDevices && done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
    const cudaError_t e = set();
    if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done[dev].store(true, std::memory_order_release);
    return e;
  }
};

// Page geometry for the cache's code widths (the HQ_PAGE_SUBPOS layout).
struct PageGeo {
  int kb, vb;    // code bits of K and V
  int pr;        // positions per sub-page
  int sub;       // bytes per sub-page
  int mask;      // offset of the bitmap words (the first-VL row follows at + 8)
  int bytes;     // bytes per page
};
__host__ __device__ __forceinline__ int kbits_of(const hq_cache& c) { return c.k_bits ? c.k_bits : 4; }
__host__ __device__ __forceinline__ int vbits_of(const hq_cache& c) { return c.v_bits ? c.v_bits : 4; }
__host__ __device__ __forceinline__ PageGeo page_geo(int kb, int vb) {
  PageGeo g;
  g.kb = kb;
  g.vb = vb;
  g.pr = HQ_PAGE_SUBPOS(kb, vb);
  g.sub = HQ_PAGE_SUBBYTES(kb, vb);
  g.mask = HQ_PAGE_MASK_OFF(kb, vb);
  g.bytes = HQ_PAGE_BYTES_KV(kb, vb);
  return g;
}
__host__ __device__ __forceinline__ PageGeo page_geo(const hq_cache& c) { return page_geo(kbits_of(c), vbits_of(c)); }

// State row of sequence b.
__host__ __device__ __forceinline__ int32_t* state_row(const hq_cache& c, int b) { return c.state + b * HQ_STATE_WORDS; }

// Pool index of page j (positions 64 j .. 64 j + 63) of (b, kv head) bh: the
// dense layout when there is no page table, else the table entry; -1 when the
// entry lies outside the pool.
__device__ __forceinline__ long long page_index(const hq_cache& c, size_t bh, int j) {
  const size_t npg = static_cast<size_t>(c.cap / HQ_PAGE_POSITIONS);
  if (c.page_table == nullptr) return static_cast<long long>(bh * npg + j);
  const int idx = c.page_table[bh * npg + j];
  return (idx >= 0 && idx < c.n_pages) ? idx : -1;
}

// K4V4 page of position p of (b, kv head) bh, for readers: an entry outside the
// pool reads pool page 0 instead (memory-safe) and flags HQ_DEVERR_PAGE.
__device__ __forceinline__ uint8_t* page_of(const hq_cache& c, size_t bh, int p) {
  const long long idx = page_index(c, bh, p >> 6);
  if (idx < 0) {
    atomicOr(reinterpret_cast<unsigned int*>(state_row(c, static_cast<int>(bh / c.Hkv)) + HQ_STATE_ERR), HQ_DEVERR_PAGE);
    return c.pages;
  }
  return c.pages + static_cast<size_t>(idx) * page_geo(c).bytes;
}

// The same for writers: null for an entry outside the pool (flagged; the caller skips the write).
__device__ __forceinline__ uint8_t* page_for_write(const hq_cache& c, size_t bh, int p) {
  const long long idx = page_index(c, bh, p >> 6);
  if (idx < 0) {
    atomicOr(reinterpret_cast<unsigned int*>(state_row(c, static_cast<int>(bh / c.Hkv)) + HQ_STATE_ERR), HQ_DEVERR_PAGE);
    return nullptr;
  }
  return c.pages + static_cast<size_t>(idx) * page_geo(c).bytes;
}
// codes (16 * bits bytes) of position p (K: which = 0, V: 1) inside its page
__host__ __device__ __forceinline__ uint8_t* row_codes(const PageGeo& pg, uint8_t* page, int which, int p) {
  const int r = p & 63, rr = r % pg.pr;
  uint8_t* sp = page + (r / pg.pr) * pg.sub;
  return which ? sp + pg.pr * 16 * pg.kb + rr * 16 * pg.vb : sp + rr * 16 * pg.kb;
}
// the 4 (scale | zero << 16) words of position p
__host__ __device__ __forceinline__ uint32_t* row_sz(const PageGeo& pg, uint8_t* page, int which, int p) {
  const int r = p & 63, rr = r % pg.pr;
  uint8_t* sp = page + (r / pg.pr) * pg.sub;
  return reinterpret_cast<uint32_t*>(sp + pg.pr * 16 * (pg.kb + pg.vb) + (which ? pg.pr * 16 : 0) + rr * 16);
}
__host__ __device__ __forceinline__ uint32_t* page_mask(const PageGeo& pg, uint8_t* page) {
  return reinterpret_cast<uint32_t*>(page + pg.mask);
}
__host__ __device__ __forceinline__ int32_t* page_vlbase(const PageGeo& pg, uint8_t* page) {
  return reinterpret_cast<int32_t*>(page + pg.mask + 8);
}

// release / acquire fences at GPU scope (cheaper than the sequentially
// consistent fence behind __threadfence)
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
// atomic add with acquire-release semantics at gpu scope (a completion ticket:
// releases what this CTA did before it, acquires what earlier ticket holders did)
__device__ __forceinline__ unsigned int atom_add_acq_rel_gpu(unsigned int* p, unsigned int v) {
  unsigned int r;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(r) : "l"(p), "r"(v) : "memory");
  return r;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void set_err(int32_t* state, uint32_t bit) {
  atomicOr(reinterpret_cast<unsigned int*>(state + HQ_STATE_ERR), bit);
}

// ----------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// non-blocking probe of a phase (no suspend hint)
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with the given parity to complete; gives up after about
// one second, sets HQ_DEVERR_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* state) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > 1000000000ull) {
      set_err(state, HQ_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// ----------------------------------------------------------------- bulk copies

// 1-D bulk copy global -> shared (no multicast), completion counted on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// L2 prefetch of a global range (a hint: no completion, no ordering); address
// and size multiples of 16 bytes
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ----------------------------------------------------------------- tensor-core helpers

// D = A(16x16, row) * B(16x8, col) + D ; f16 inputs, f32 accumulate.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose an 8x8 b16 tile held one 32-bit pair per thread.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Programmatic dependent launch (sm_90+): wait until the grids this one depends
// on have completed and their writes are visible / allow the next grid in the
// stream to begin launching.  Both are no-ops for a normal launch.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// (a & b) | c as one LOP3
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

__device__ __forceinline__ uint32_t hfma2_u(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

__device__ __forceinline__ uint32_t hsub2_u(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Nibble -> fp16 via the exponent-bias trick: OR-ing a 4-bit value n into the
// mantissa of 1024.0 (0x6400) gives 1024 + n exactly; subtracting 1024 leaves n.
// lo: nibbles at bits 0..3 and 16..19 of w; hi: nibbles at bits 4..7 and 20..23
// (they land as 1024 + 16 n, scaled back by 1/16 and shifted by -64, exact).
constexpr uint32_t MAGIC = 0x64006400u;      // (1024, 1024)
constexpr uint32_t H2_1024 = 0x64006400u;
constexpr uint32_t H2_SIXTEENTH = 0x2C002C00u;  // (1/16, 1/16)
constexpr uint32_t H2_M64 = 0xD400D400u;        // (-64, -64)

__device__ __forceinline__ uint32_t nib_lo(uint32_t w) { return hsub2_u(and_or(w, 0x000F000Fu, MAGIC), H2_1024); }
__device__ __forceinline__ uint32_t nib_hi(uint32_t w) {
  return hfma2_u(and_or(w, 0x00F000F0u, MAGIC), H2_SIXTEENTH, H2_M64);
}

}  // namespace hq
