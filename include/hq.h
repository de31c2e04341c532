/*
 * hq.h — C ABI of libhq.so: hybrid-precision attention on NVIDIA B200 (sm_100a).
 *
 * What the library computes is the hot path of HyQuant ("HyQuant:
 * Hybrid-Precision Quantization for LLM Attention"):
 *
 *   - keys are split three ways: vertical-line (VL) positions and a recent
 *     window stay FP16, every other position is stored 4-bit (K4V4)
 *     (agihunt.info digest of the paper, method paragraph; repository README,
 *     Overview);
 *   - decode attention runs over that hybrid cache with dequantisation fused
 *     into the online-softmax KV scan, so no FP16 copy of the cache is ever
 *     materialised (digest, prefill/decode paragraph; README Overview item 3);
 *   - the VL set is the top-rho (default 5 %) of the non-window prefix by
 *     accumulated column attention mass, re-identified every 64 tokens from at
 *     most 64 buffered FP16 queries (digest, method paragraph; README Overview
 *     item 1 and "Overhead");
 *   - new tokens are staged and merged into the hybrid layout later (digest,
 *     prefill/decode paragraph);
 *   - prefill is one FlashAttention-style causal pass whose quantised tiles run
 *     on low-precision tensor cores while VL and window tiles stay FP16, under a
 *     single online softmax (digest, prefill/decode paragraph; README Overview
 *     item 2).
 *
 * K4V4 layout (the pages name the format but print no layout; this library
 * fixes it): per token and head, D = 128 values in 4 groups of 32;
 * scale = fp16(fp32(max - min) / 15), zero = min (fp16);
 * q = clamp(rint_even((x - zero) / scale), 0, 15) with float32 RN arithmetic
 * (q = 0 when scale == 0); two nibbles per byte, low nibble first; the
 * dequantised value is zero + q * scale.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers, 16-byte aligned, owned by the
 *     caller; the library allocates nothing.  Its only state is the last error
 *     message of each host thread (hq_last_error) and, for
 *     hq_decode_attn_noalloc alone, a fixed device scratch array of its own.
 *   - fp16 tensors are passed as uint16_t* (IEEE binary16 bit patterns).
 *   - Calls are asynchronous on `stream`.  Arguments are validated on the host
 *     before anything is launched; on a non-HQ_OK status nothing was launched.
 *   - Conditions that depend on device-resident lengths (a full staging area,
 *     an exhausted capacity) cannot be seen by the host: the kernels skip their
 *     work and OR a HQ_DEVERR_* bit into state[b][HQ_STATE_ERR] of the sequence
 *     concerned; read it after synchronising.  No kernel traps or spins
 *     without a bound.
 *   - Sequences are independent: each batch row b has its own lengths (a row
 *     of the state array), so one call serves a batch of sequences of
 *     different lengths.  The K4V4 store may be paged (page_table), so that the
 *     pages of a sequence need not be contiguous.  A single sequence is
 *     addressed by a descriptor whose pointers are offset to its row (B = 1),
 *     e.g. to install its prefix while the others keep decoding.
 */
#ifndef HQ_H
#define HQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HQ_ABI_VERSION 4
#define HQ_HEAD_DIM 128       /* D: the only head size built */
#define HQ_GROUP 32           /* K4V4 group length along D */
#define HQ_STAGE 64           /* staged tokens before a merge = reselection period */
#define HQ_QBUF 64            /* buffered queries kept for the column-mass estimate */
#define HQ_MAX_GQA 8          /* query heads per kv head supported by the decode kernel */
/* K4V4 store page: 64 positions of one (batch, kv head), one contiguous block */
#define HQ_PAGE_POSITIONS 64
#define HQ_PAGE_BYTES 10304
#define HQ_PAGE_KCODES 0        /* [64][D/2] K codes, row r = position 64 j + r */
#define HQ_PAGE_VCODES 4096     /* [64][D/2] V codes */
#define HQ_PAGE_KSZ 8192        /* [64][D/32] uint32 K (scale bits | zero bits << 16) */
#define HQ_PAGE_VSZ 9216        /* [64][D/32] uint32 V (scale | zero << 16) */
#define HQ_PAGE_VLMASK 10240    /* 2 uint32: bit r of word r/32 <=> position 64 j + r is a vertical line */
#define HQ_PAGE_VLBASE 10248    /* int32: VL-store row of the page's first vertical line (valid when the bitmap is non-zero) */
/* Other code widths (k_bits, v_bits in {2, 4, 8}; README Mode reference: K8V8,
 * K4V2, K2V4 beside K4V4).  Same scale/zero rule with 2^bits - 1 levels and
 * 8 / bits codes per byte, lowest bits first.  A page of 64 positions is cut
 * into sub-pages of HQ_PAGE_SUBPOS(kb, vb) positions (64, or 32 when kb + vb >
 * 8), each laid out [K codes][V codes][K (scale|zero) words][V words] with
 * 16 * bits bytes of codes per position; the bitmap and the first-VL row follow
 * the sub-pages.  For kb = vb = 4 this is exactly the HQ_PAGE_* layout above. */
#define HQ_PAGE_SUBPOS(kb, vb) (((kb) + (vb)) > 8 ? 32 : 64)
#define HQ_PAGE_SUBBYTES(kb, vb) (HQ_PAGE_SUBPOS(kb, vb) * (16 * (kb) + 16 * (vb) + 32))
#define HQ_PAGE_MASK_OFF(kb, vb) ((64 / HQ_PAGE_SUBPOS(kb, vb)) * HQ_PAGE_SUBBYTES(kb, vb))
#define HQ_PAGE_BYTES_KV(kb, vb) (((HQ_PAGE_MASK_OFF(kb, vb) + 16) + 63) / 64 * 64)
/* FP16 ring length for a window W: W + HQ_STAGE rounded up to a multiple of 16 */
#define HQ_RING_LEN(W) ((((W) + HQ_STAGE) + 15) / 16 * 16)

typedef struct CUstream_st* hq_stream_t;  /* same type as cudaStream_t */

#if defined(__GNUC__)
#define HQ_API __attribute__((visibility("default")))
#else
#define HQ_API
#endif

typedef enum hq_status {
  HQ_OK = 0,
  HQ_ERR_INVALID = 1,      /* null/misaligned pointer, bad shape or argument */
  HQ_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement (e.g. D != 128) */
  HQ_ERR_WORKSPACE = 3,    /* workspace missing or smaller than hq_*_workspace_bytes() */
  HQ_ERR_CAPACITY = 4,     /* a host-visible size exceeds the cache's capacity */
  HQ_ERR_CUDA = 5          /* a CUDA runtime call or launch failed */
} hq_status;

/* device-side error bits, OR-ed into state[b][HQ_STATE_ERR] */
#define HQ_DEVERR_STAGING_FULL 0x1u  /* decode with HQ_STAGE tokens staged: select + merge first */
#define HQ_DEVERR_CAPACITY 0x2u      /* T would exceed cap */
#define HQ_DEVERR_VL_CAPACITY 0x4u   /* k = ceil(rho * n) exceeds vl_cap (clamped) */
#define HQ_DEVERR_TIMEOUT 0x8u       /* a bounded wait gave up (never expected) */
#define HQ_DEVERR_PAGE 0x10u         /* a page-table entry outside [0, n_pages): pool page 0 was read
                                        instead (the outputs of that sequence are unspecified) and
                                        nothing was written through the entry */

/* words of one sequence's row of the device-resident state (int32[B][HQ_STATE_WORDS]) */
enum {
  HQ_STATE_T = 0,         /* current length: positions 0 .. T-1 are cached */
  HQ_STATE_NPACKED = 1,   /* positions 0 .. n_packed-1 have a K4V4 record */
  HQ_STATE_NVL = 2,       /* rows in the VL store */
  HQ_STATE_NQ = 3,        /* valid buffered queries (<= HQ_QBUF) */
  HQ_STATE_KSEL = 4,      /* entries written to vl_sel by the last hq_select_vlines */
  HQ_STATE_ERR = 5,       /* HQ_DEVERR_* bits */
  HQ_STATE_WORDS = 8
};

/*
 * The hybrid KV cache of one attention layer.  Every array is caller-owned
 * device memory laid out as stated ([..] = row-major shape, innermost last).
 * R = HQ_RING_LEN(W) is the FP16 ring length (W + HQ_STAGE rounded up to 16).
 *
 *   pages     uint8  [B, Hkv, cap/64, PB]  (page_table == NULL) or a page pool uint8 [n_pages, PB]
 *             (page_table != NULL), PB = HQ_PAGE_BYTES_KV(k_bits, v_bits): the packed store, one page per
 *             64 positions (layout HQ_PAGE_* for K4V4, sub-pages for the other widths): codes
 *             of both K and V, their per-group (scale, zero) words and the VL bitmap of the
 *             page's positions, so that one contiguous copy brings a whole (sub-)page on chip,
 *             then the VL-store row of the page's first vertical line (at
 *             HQ_PAGE_MASK_OFF(k_bits, v_bits) + 8); the bytes after it up to PB are padding
 *   kf, vf    fp16   [B, Hkv, vl_cap, D]  VL store rows, in vl_pos order
 *   vl_pos    int32  [B, Hkv, vl_cap]     VL positions, ascending (first n_vl valid)
 *   kr, vr    fp16   [B, Hkv, R, D]       recent window + staging; position p at slot p % R
 *   qbuf      fp16   [B, Hq, HQ_QBUF, D]  buffered decode queries; position p at slot p % HQ_QBUF
 *   vl_sel    int32  [B, Hkv, vl_cap]     output of hq_select_vlines, input of hq_pack_merge
 *   state     int32  [B, HQ_STATE_WORDS]  device-resident lengths of each sequence (HQ_STATE_*)
 *   page_table int32 [B, Hkv, cap/64]    optional (NULL: pages is the dense [B, Hkv, cap/64, ..]
 *             array): entry (b, h, j) is the pool page holding positions 64 j .. 64 j + 63
 *             of sequence b, kv head h; 4-byte aligned; entries of pages no position
 *             reaches are not read.  Pages of different (b, h) must be distinct.
 *   score_acc float [B, Hkv, cap]        optional running column-mass scores (NULL: each
 *             reselection ranks its own column mass).  When set, the prefix selection
 *             (init mode) stores its column mass there (zero past the scored prefix) and
 *             every decode-mode reselection adds its column mass to it and ranks the sums
 *             (README Overview item 1, "running column-mass score").
 *   qlse      float [B, Hq, HQ_QBUF]     optional (NULL: not kept): each decode step stores the
 *             log-sum-exp (base 2, over its T + 1 logits q.k / sqrt(D)) of its query next to
 *             the query itself (slot T % HQ_QBUF).  A decode-mode reselection whose buffered
 *             queries all came after the last merge (so they saw the keys exactly as the
 *             reselection does) takes its row normalisers from here instead of a first
 *             pass over the keys.  Decode steps with sm_scale != 1/sqrt(D) store NaN.
 *
 * Limits checked by hq_cache_validate(): D == 128; Hq % Hkv == 0 and
 * Hq / Hkv <= HQ_MAX_GQA; W >= 0; 0 <= rho_bp <= 10000; cap a positive
 * multiple of 128; vl_cap a positive multiple of 16; with a page table,
 * n_pages >= 1; (k_bits, v_bits) one of (4, 4), (8, 8), (4, 2), (2, 4).
 * Pages are HQ_PAGE_BYTES_KV(k_bits, v_bits) bytes.
 * Fields W and rho_bp fix the method's window and VL ratio (basis points:
 * 500 = 5 %).  The fp16 positions in [n_packed, T) live in the ring, VL rows
 * in kf/vf, every other position < n_packed is read from its K4V4 record.
 */
typedef struct hq_cache {
  int32_t B, Hq, Hkv, D;
  int32_t W, rho_bp, cap, vl_cap;
  uint8_t* pages;
  uint16_t* kf;
  uint16_t* vf;
  int32_t* vl_pos;
  uint16_t* kr;
  uint16_t* vr;
  uint16_t* qbuf;
  int32_t* vl_sel;
  int32_t* state;
  int32_t* page_table;
  float* score_acc;
  float* qlse;
  int32_t n_pages;
  int32_t k_bits;     /* code bits of packed keys: 4 (0 means 4), 8 or 2 */
  int32_t v_bits;     /* code bits of packed values: 4 (0 means 4), 8 or 2 */
  int32_t reserved;   /* 0 */
} hq_cache;

/* Operation codes for hq_workspace_bytes. */
enum { HQ_OP_SELECT = 0, HQ_OP_MERGE = 1, HQ_OP_DECODE = 2 };

HQ_API int32_t hq_abi_version(void);
HQ_API const char* hq_status_str(hq_status s);

/* After a call returned HQ_ERR_CUDA: which step failed and the CUDA error name
 * (e.g. "prefill launch: cudaErrorLaunchOutOfResources").  Per host thread;
 * the string stays valid until the next failing call on that thread. */
HQ_API const char* hq_last_error(void);

/* Host-side check of a cache descriptor (shapes, limits, 16-byte alignment of
 * every pointer).  Returns HQ_OK or HQ_ERR_INVALID / HQ_ERR_UNSUPPORTED. */
HQ_API hq_status hq_cache_validate(const hq_cache* c);

/* Bytes of device workspace an operation needs for this cache; `L` is the
 * prefix length for an init-mode select/merge (ignored otherwise).
 * HQ_OP_DECODE and HQ_OP_MERGE workspaces start with completion counters:
 * zero-fill the workspace once before its first use; the kernels return the
 * counters to zero at the end of every call.  A workspace must not be shared
 * by calls that can run at the same time. */
HQ_API size_t hq_workspace_bytes(const hq_cache* c, int32_t op, int32_t L);

/*
 * Reset every sequence of the descriptor to empty: its state row to 0, the
 * VL bitmap of each of its pages (through the page table, if any) cleared and
 * its running scores (score_acc, if any) zeroed.
 */
HQ_API hq_status hq_cache_reset(const hq_cache* c, hq_stream_t stream);

/*
 * Vertical-line selection (digest, method paragraph; README Overview item 1).
 * For every (b, kv head): column mass
 *     score_j = sum over the group's query heads h and buffered queries i of
 *               softmax_{j' <= p_i}(q_{h,i} . k_{j'} * sm_scale)[j],
 * for j in the non-window prefix [0, n), n = T - W, sm_scale = 1/sqrt(D);
 * then the k = ceil(n * rho_bp / 10000) largest scores (ties -> lower
 * position) are written to c->vl_sel in ascending position order and k to
 * state[b][HQ_STATE_KSEL]; every sequence b uses its own T, n and k.
 *
 * Init mode (k_dense != NULL): keys are the dense FP16 prefix
 *   k_dense [B, Hkv, L, D], T = L; queries q_ext [B, Hq, nq, D] sit at
 *   positions L-nq .. L-1 (1 <= nq <= HQ_QBUF, nq <= L).  The cache's state
 *   is not read.
 * Decode mode (k_dense == NULL, q_ext == NULL): keys are the cache in its
 *   current representation (VL rows FP16, other packed positions
 *   dequantised, ring FP16), T and the buffered queries come from state/qbuf.
 * scores_out (optional, may be NULL): float [B, Hkv, cap] receives the scores
 *   (entries >= n are unspecified).
 * Errors: HQ_ERR_INVALID for bad pointers/shapes; k > vl_cap is clamped and
 *   flagged with HQ_DEVERR_VL_CAPACITY.
 */
HQ_API hq_status hq_select_vlines(const hq_cache* c, const uint16_t* k_dense, int32_t L,
                           const uint16_t* q_ext, int32_t nq, float* scores_out,
                           void* ws, size_t ws_bytes, hq_stream_t stream);

/*
 * Staging -> hybrid merge (digest, prefill/decode paragraph).
 * Init mode (k_dense, v_dense != NULL, both [B, Hkv, L, D] FP16): install a
 *   prefix of L tokens: positions [0, L-W) get their K4V4 records, the last
 *   min(W, L) positions go to the ring, the VL store is filled from c->vl_sel
 *   (state[b][HQ_STATE_KSEL] entries, FP16 rows taken from the dense prefix);
 *   every row b of state becomes T = L, n_packed = max(L-W, 0), n_q = 0.
 *   Requires L <= cap.  Sequences of different prefix lengths are installed
 *   one at a time through single-sequence descriptors.
 * Merge mode (both NULL): positions [n_packed, T-W) leave the window and get
 *   their K4V4 records; the VL store is rebuilt from c->vl_sel: a row keeps the
 *   position's current FP16 value when it has one (old VL row or ring),
 *   otherwise it is the dequantised record rounded once to FP16; n_packed
 *   becomes max(n_packed, T-W).  Records are never rewritten.  Each sequence
 *   uses its own lengths.
 */
HQ_API hq_status hq_pack_merge(const hq_cache* c, const uint16_t* k_dense, const uint16_t* v_dense,
                        int32_t L, void* ws, size_t ws_bytes, hq_stream_t stream);

/*
 * One decode step (digest, prefill/decode paragraph; README Overview item 3):
 * append k_new, v_new [B, Hkv, D] at position T (ring) and q [B, Hq, D] to
 * the query buffer, then
 *     out[b, h] = softmax(q[b,h] . K^T * sm_scale) V
 * over all T+1 positions, each key/value in its stored representation
 * (dequantisation fused into the scan; split-K over the sequence with a
 * log-sum-exp merge).  out: fp16 [B, Hq, D].  Increments T.  Every sequence
 * b attends over its own T_b + 1 positions.
 * If HQ_STAGE tokens of sequence b are already staged (T - n_packed == W +
 * HQ_STAGE) or T == cap, nothing of that sequence is written (its out rows
 * included) and HQ_DEVERR_STAGING_FULL / _CAPACITY is set in its state row;
 * the other sequences proceed.  B * Hkv <= 2048 (else HQ_ERR_UNSUPPORTED).
 * After a HQ_DEVERR_TIMEOUT the workspace's counters may not be zero: zero
 * the workspace again before the next call.
 */
HQ_API hq_status hq_decode_attn(const hq_cache* c, const uint16_t* q, const uint16_t* k_new,
                         const uint16_t* v_new, uint16_t* out, float sm_scale,
                         void* ws, size_t ws_bytes, hq_stream_t stream);

/*
 * Hybrid causal prefill (digest, prefill/decode paragraph; README Overview
 * item 2, modes "vquant_vert" / "hybrid_full"): for query i and key j <= i,
 *   j is a window key if i - W < j <= i, else a VL key if j is in vl_pos[b, kvh],
 *   else a quantised key;
 * window and VL keys use FP16 Q, K, V; quantised keys use, by qk_format,
 *   HQ_PREFILL_E4M3:    FP8 e4m3 Q, K, V with one float32 scale per (b, head,
 *                       128 positions) (scale = amax / 448, values stored as
 *                       e4m3_RN_sat(x / scale));
 *   HQ_PREFILL_INT8_QK: INT8 Q, K with one float32 scale per (b, head, 128
 *                       positions) (scale = amax / 127, codes
 *                       clamp(rint_even(x / scale), -127, 127)) and FP16 V
 *                       (README Overview item 2, the INT8-QK / FP16-PV kernels);
 * one softmax covers all three classes.
 *   q [B, Hq, L, D], k, v [B, Hkv, L, D], out [B, Hq, L, D]: fp16
 *   vl_pos int32 [B, Hkv, vl_stride], first n_vl entries ascending, < L
 *     (0 <= n_vl <= min(vl_stride, L))
 * Workspace: at least hq_prefill_workspace_bytes(B, Hq, Hkv, L, D, vl_stride)
 * bytes, 16-byte aligned; one call's workspace must not be shared with a call
 * that can run at the same time.  It holds, in this order (each region starting
 * on a 1024-byte boundary, Lp = L rounded up to a multiple of 128):
 *   bytes [0, 4)  uint32 error word, cleared by the call: non-zero when a
 *                 bounded wait of the kernel gave up (never expected; the
 *                 output is then incomplete); read it after synchronising;
 *   e4m3 (or INT8) codes of Q [B, Hq, Lp, D], e4m3 (or INT8) codes of K
 *   [B, Hkv, Lp, D], fp16 values fp16(fp32(e4m3(V / scale)) * scale) of V
 *   [B, Hkv, Lp, D] (e4m3 format only), then the per-block scales and gathered
 *   VL rows (internal).
 * Rows past L of the three coded tensors are zero.
 */
HQ_API size_t hq_prefill_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t L, int32_t D, int32_t vl_stride);
enum { HQ_PREFILL_E4M3 = 0, HQ_PREFILL_INT8_QK = 1 };
HQ_API hq_status hq_prefill_attn(int32_t B, int32_t Hq, int32_t Hkv, int32_t L, int32_t D,
                          const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          const int32_t* vl_pos, int32_t n_vl, int32_t vl_stride, int32_t W,
                          int32_t qk_format, float sm_scale, uint16_t* out, void* ws, size_t ws_bytes,
                          hq_stream_t stream);

/*
 * Allocation-free decode step.  The paper has no counterpart: this is a
 * deployment variant of hq_decode_attn for callers that may not allocate
 * device memory at all, such as a plugin inside a serving engine that owns all
 * device memory, or a latency-critical loop where cudaMalloc / cudaFree would
 * synchronise the device.  Arguments and result are those of hq_decode_attn,
 * minus the workspace: the library uses a fixed scratch array of
 * HQ_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until the
 * process exits.
 *   - The first call on a device (with that device current) looks up the
 *     array's device address; make that first call before any stream capture.
 *     After the device is reset (cudaDeviceReset, or its primary context
 *     released and created again) the next call sees a new context and looks
 *     the address up again: make that call before any capture as well.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents; each call clears what must start at zero itself.  Calls whose
 *     executions can overlap on the GPU (unordered streams) race on the array:
 *     order them on one stream.
 *   - Returns HQ_ERR_WORKSPACE when this cache's decode workspace
 *     (hq_workspace_bytes(c, HQ_OP_DECODE, 0)) exceeds HQ_NOALLOC_SCRATCH_BYTES;
 *     nothing is launched then.  It never calls cudaMalloc or cudaFree.
 */
#define HQ_NOALLOC_SCRATCH_BYTES (4u << 20)
HQ_API hq_status hq_decode_attn_noalloc(const hq_cache* c, const uint16_t* q, const uint16_t* k_new,
                                        const uint16_t* v_new, uint16_t* out, float sm_scale, hq_stream_t stream);

/*
 * Measurement helper (no counterpart in the method): reads `bytes` (a multiple
 * of 16) of device memory at `src` (16-byte aligned) with 16-byte streaming
 * loads from sms * ctas_per_sm CTAs of 512 threads (1 <= ctas_per_sm <= 4),
 * and XORs what it read into *sink (device, 4-byte aligned) so the loads are
 * kept.  Timing it over a buffer far larger than L2 gives the read-only HBM
 * bandwidth ceiling that a scan such as the decode step can approach.
 */
HQ_API hq_status hq_diag_stream_read(const void* src, size_t bytes, uint32_t* sink, int32_t ctas_per_sm,
                                     hq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H */
