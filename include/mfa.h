/*
 * mfa.h -- mask-aware flash attention (forward pass and gradients) for NVIDIA
 * B200 (sm_100a).
 *
 * C ABI of libmfa.so. Two calls carry the forward computation:
 *
 *   mfa_build_tile_map  reduces a compact mask description to a per-tile
 *                       SKIP / FULL / PARTIAL map plus, for every query tile,
 *                       the ascending list of key tiles that must be computed
 *                       (Binary Block Masking, "Efficiently Dispatching Flash
 *                       Attention For Partially Filled Attention Masks",
 *                       abstract: fully masked blocks are never processed and
 *                       fully visible blocks need no per-element mask).
 *   mfa_fwd             computes out = softmax(Q K^T / sqrt(d) + mask) V and the
 *                       natural-log log-sum-exp of every query row, visiting
 *                       only the listed key tiles (FlashMask author response:
 *                       calculations for fully masked blocks are unnecessary).
 *   mfa_bwd             computes dq, dk, dv through the same map (FlashMask's
 *                       masks serve training first, per the author response).
 *   mfa_decode          attends a few query rows to selected 64-key blocks of a
 *                       long cache, split over CTAs (the selected-key flash
 *                       attention pull request).
 * mfa_fwd_bias adds an ALiBi bias to mfa_fwd, mfa_mask_from_sparse_mode turns
 * an Ascend sparse mode into a mask description, and mfa_fwd_noalloc runs the
 * map build and forward pass without any buffer from the caller but the tensors.
 *
 * Conventions shared by every call:
 *
 * - All tensor and array pointers are DEVICE pointers unless a comment says
 *   otherwise. The caller allocates and owns every buffer; the library
 *   allocates no device memory. Between calls it keeps only the record of
 *   the devices on which it has set each kernel's shared-memory attribute,
 *   and mfa_fwd_noalloc's static scratch array (part of the module).
 * - Every call launches on the CURRENT CUDA device (cudaSetDevice), which must
 *   be the device that holds the call's tensors and arrays, and `stream` must
 *   belong to that device. The library does not switch devices itself.
 * - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *   is the legacy default stream). Argument errors are detected on the host and
 *   returned before anything is launched. Problems only the device can see
 *   (bounds out of range, a bounded wait that gave up) are recorded in the tile
 *   map's error word and reported by mfa_get_device_status.
 * - Combinations the kernels do not implement return MFA_ERR_UNSUPPORTED; the
 *   library never computes a silently different mask (the selected-key pull
 *   request's lesson: a kernel must decline an op it cannot compute exactly).
 *
 * Mask semantics (masked = not attended):
 * - COLWISE, FlashMask-style column-wise row intervals: for key column j, query
 *   rows i with lts[j] <= i < lte[j] or uts[j] <= i < ute[j] are masked.
 *   Half-open; start >= end is empty; every bound must lie in [0, Nq]. Arrays
 *   are int32 [B, Hm, Nk], contiguous. A NULL pair (lts/lte or uts/ute) is the
 *   empty interval. A causal mask is given explicitly as uts = 0, ute = j.
 * - BAND, Ascend sparseMode 0 (equal to sparseMode 4 when Nq == Nk): the pair
 *   (i, j) is attended iff -pre_tokens <= j - i <= next_tokens, both ends
 *   inclusive (Ascend CANN "sparseMode introduction", sparseMode 0 and 4).
 * - BLOCKSEL, per-query-block key-block lists (the selected-key flash attention
 *   pull request): sel is int32 [B, Hm, ceil(Nq/64), sel_k]; entry -1 is no
 *   entry, duplicates count once, entries must lie in [-1, ceil(Nk/64)).
 *   Query i attends key j iff block j/64 is listed for block i/64 and j <= i.
 * A query row that attends no key gets out = 0 and lse = -inf.
 */
#ifndef MFA_H_
#define MFA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MFA_ABI_VERSION 1

typedef enum {
  MFA_OK = 0,
  MFA_ERR_INVALID_ARG = 1,    /* NULL pointer, negative size, bad enum value   */
  MFA_ERR_UNSUPPORTED = 2,    /* a valid combination the kernels do not cover */
  MFA_ERR_SHAPE_MISMATCH = 3, /* tensors, mask and map disagree on a size      */
  MFA_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed          */
  MFA_ERR_DEVICE = 5          /* the device recorded an error (see error bits) */
} mfa_status;

typedef enum { MFA_BF16 = 0, MFA_F32 = 1 } mfa_dtype;

typedef enum { MFA_MASK_COLWISE = 0, MFA_MASK_BAND = 1, MFA_MASK_BLOCKSEL = 2 } mfa_mask_kind;

/* Device error word bits (mfa_tile_map.err). */
#define MFA_DEVERR_BOUNDS 1u   /* a column bound outside [0, Nq]                      */
#define MFA_DEVERR_SEL 2u      /* a selection entry outside [-1, ceil(Nk/64))         */
#define MFA_DEVERR_TIMEOUT 4u  /* a bounded wait in mfa_fwd / mfa_bwd gave up; outputs invalid */
#define MFA_DEVERR_MAP 8u      /* mfa_fwd read a tile list entry outside [0, nkt)     */

/* A 4-D tensor [B, H, N, D]; strides in ELEMENTS, stride[3] must be 1. */
typedef struct {
  void* data;        /* device pointer                                    */
  int32_t dtype;     /* mfa_dtype                                         */
  int32_t reserved;
  int64_t B, H, N, D;
  int64_t stride[4];
} mfa_tensor;

/* The tile map: shape fields are set by mfa_tile_map_init, the pointers carve
 * one caller-owned device buffer of mfa_tile_map_bytes() bytes. Layout (per
 * batch b, mask head hm; nqt = ceil(Nq/block_q), nkt = ceil(Nk/block_k)):
 *   kminmax    int32 [B, Hm, nkt, 8]  min/max over the k-tile's columns of
 *              LTS, LTE, UTS, UTE (in that order, min then max), with every
 *              empty interval written as start = Nq, end = 0; the band kind is
 *              first turned into UT = [0, clamp(j - next, 0, Nq)),
 *              LT = [clamp(j + pre + 1, 0, Nq), Nq). Zero for BLOCKSEL.
 *   tile_class uint8 [B, Hm, nqt, nkt] bits 0-1: 0 SKIP, 1 FULL, 2 PARTIAL.
 *              BLOCKSEL only: bit 4 + 2*qs + ks set when 64x64 sub-block
 *              (qs, ks) of the tile holds a visible pair.
 *   tile_list  int32 [B, Hm, nqt, nkt] ascending non-SKIP k-tiles, -1 padded.
 *   tile_count int32 [B, Hm, nqt].
 *   order      int32 [B*Hm*nqt] flat (b, hm, qt) sorted by count, largest
 *              first, ties by index (the forward pass's work order).
 *   err        uint32 [4]: err[0] is the device error word (MFA_DEVERR_*
 *              bits), set by mfa_build_tile_map and mfa_fwd; err[1] and
 *              err[2] are mfa_fwd's work counters (the next work item and the
 *              number of finished CTAs), err[3] mfa_build_tile_map's count of
 *              finished classification blocks; the counters are left at zero
 *              after every call. All four are cleared by mfa_build_tile_map. Because of the
 *              counters, mfa_fwd calls that share one map must not overlap on
 *              the GPU (issue them on one stream, or order the streams).
 * Class rule for COLWISE / BAND with r0 = qt*block_q, r1 = min(r0+block_q, Nq):
 *   SKIP    if (LTSmax <= r0 && LTEmin >= r1) || (UTSmax <= r0 && UTEmin >= r1)
 *   FULL    else if (LTSmin >= r1 || LTEmax <= r0) && (UTSmin >= r1 || UTEmax <= r0)
 *   PARTIAL otherwise.
 * BLOCKSEL: SKIP if every valid 64x64 sub-block is unlisted or above the
 * diagonal block, FULL if every one is listed and strictly below it. */
typedef struct mfa_tile_map {
  int32_t B, Hm, Nq, Nk, block_q, block_k, nqt, nkt;
  int32_t kind;      /* mask kind of the last mfa_build_tile_map (-1 before) */
  int32_t reserved;
  int32_t* kminmax;
  uint8_t* tile_class;
  int32_t* tile_list;
  int32_t* tile_count;
  int32_t* order;
  uint32_t* err;
} mfa_tile_map;

/* A compact mask description. Sizes: B batch, Hm mask heads (1 = one mask
 * shared by all query heads, or Hq = one per query head), Nq queries, Nk keys. */
typedef struct {
  int32_t kind;                   /* mfa_mask_kind                            */
  int32_t B, Hm, Nq, Nk;
  int32_t sel_k;                  /* BLOCKSEL: entries per query block        */
  int32_t sel_block;              /* BLOCKSEL: must be 64                     */
  int32_t reserved;
  const int32_t *lts, *lte, *uts, *ute; /* COLWISE: device int32 [B, Hm, Nk]  */
  int64_t pre_tokens, next_tokens;      /* BAND                               */
  const int32_t* sel;                   /* BLOCKSEL: device int32 [B,Hm,nqb,sel_k] */
  const mfa_tile_map* map;              /* mfa_fwd: the map built from this mask */
} mfa_mask_desc;

/* ABI version of the loaded library (MFA_ABI_VERSION). Host only. */
int32_t mfa_abi_version(void);

/* Human-readable name of a status code. Host only; never NULL. */
const char* mfa_status_string(mfa_status s);

/* Bytes of device memory a tile map of this shape needs (0 on bad arguments).
 * block_q and block_k must each be 64 or 128. Host only. */
size_t mfa_tile_map_bytes(int32_t B, int32_t Hm, int32_t Nq, int32_t Nk,
                          int32_t block_q, int32_t block_k);

/* Fill `map` (host struct) with the shape and with pointers into `device_buf`
 * (caller-owned, 256-byte aligned, at least mfa_tile_map_bytes() bytes). No
 * device work. Returns INVALID_ARG / UNSUPPORTED on bad arguments. */
mfa_status mfa_tile_map_init(mfa_tile_map* map, void* device_buf, size_t bytes,
                             int32_t B, int32_t Hm, int32_t Nq, int32_t Nk,
                             int32_t block_q, int32_t block_k);

/* Ascend sparse modes (Ascend CANN "sparseMode introduction" page, one
 * paragraph per mode) as a compact mask description. Rows are queries [0, Nq), columns
 * keys [0, Nk); d = Nk - Nq.
 *   0 defaultMask   band -pre <= j - i <= next, origin at the upper left
 *   2 leftUpCausal  j <= i
 *   3 rightDownCausal  j - i <= d
 *   4 band from the lower-right vertex: -pre <= (j - i) - d <= next
 *   5, 6 prefix     j < prefix[b] or j - i <= d (6 differs from 5 only in the
 *                   page's attenMask input format)
 *   7, 8 varlen, long sequence split externally: B = 1 packs n_seq sequences
 *                   with cumulative query ends seq_q (actual_seq_qlen) and key
 *                   ends seq_kv (actual_seq_kvlen); pairs of different
 *                   sequences are masked. Inside a sequence of lengths (lq, lk):
 *                   mode 7 is rightDownCausal except the last non-empty
 *                   sequence, mode 8 leftUpCausal except the first non-empty
 *                   one, which take the band from the sequence's lower-right
 *                   vertex with (pre, next).
 * Mode 1 (a full attenMask) has no compact form: MFA_ERR_UNSUPPORTED. */
typedef struct mfa_sparse_mode {
  int32_t mode;
  int32_t reserved;                /* 0 */
  int64_t pre_tokens, next_tokens; /* modes 0, 4, 7, 8 */
  const int64_t* prefix;           /* modes 5, 6: DEVICE [B] prefix lengths */
  const int64_t* seq_q;            /* modes 7, 8: DEVICE [n_seq] cumulative query ends */
  const int64_t* seq_kv;           /* modes 7, 8: DEVICE [n_seq] cumulative key ends */
  int32_t n_seq;                   /* modes 7, 8: number of packed sequences (>= 1) */
  int32_t reserved2;               /* 0 */
} mfa_sparse_mode;

/* Fill *out (kind, B, Hm = 1, Nq, Nk and the kind's fields; out->map is left
 * NULL) for the sparse mode `sm`, the library's mask description for it.
 *   Modes 0, 2, 3, 4 become MFA_MASK_BAND with the tokens shifted to the
 *   upper-left origin (pre - d, next + d for mode 4); nothing is launched and
 *   the four arrays may be NULL.
 *   Modes 5-8 become MFA_MASK_COLWISE: one kernel writes the caller-owned
 *   DEVICE int32 arrays lts, lte, uts, ute [B, 1, Nk] on `stream` (every key
 *   column needs at most the two masked row intervals of that format). The
 *   description points at those arrays, which must outlive its use.
 *   Prefix lengths and cumulative ends are clamped to [0, Nk] / [0, Nq], and
 *   tokens to +-(Nq + Nk + 1); the cumulative ends must not decrease (the
 *   key column of a sequence is found by binary search). Keys past the last
 *   sequence are masked for every query.
 * Errors: MFA_ERR_INVALID_ARG (NULL sm/out, shapes < 0, B > 65535, B != 1 or n_seq < 1
 * for modes 7, 8, missing arrays), MFA_ERR_UNSUPPORTED (mode 1 or unknown),
 * MFA_ERR_CUDA (launch failure). */
mfa_status mfa_mask_from_sparse_mode(const mfa_sparse_mode* sm, int32_t B, int32_t Nq, int32_t Nk, int32_t* lts,
                                     int32_t* lte, int32_t* uts, int32_t* ute, mfa_mask_desc* out, void* stream);

/* Build `map` from `mask` on `stream`: clears err, computes kminmax,
 * tile_class, tile_list, tile_count and order (two kernel launches). The
 * mask's shape must equal the map's. mask->map is ignored. Device-detected
 * range errors set MFA_DEVERR_BOUNDS / MFA_DEVERR_SEL. */
mfa_status mfa_build_tile_map(const mfa_mask_desc* mask, mfa_tile_map* map, void* stream);

/* Attention forward pass on `stream`.
 *   q   [B, Hq, Nq, D], k and v [B, Hkv, Nk, D], out [B, Hq, Nq, D], all of one
 *       dtype, D in {64, 128}: MFA_BF16 runs on the bf16 tensor cores; MFA_F32
 *       runs in fp32 on the CUDA cores (tf32 tensor-core scores would move lse
 *       by ~2e-3) and writes fp32 out. Hq % Hkv == 0: query head h reads
 *       key/value head h / (Hq/Hkv).
 *       stride[3] == 1, other strides and the base address 16-byte aligned.
 *   mask  description with mask->map built from it by mfa_build_tile_map
 *         (same kind and shape); Hm must be 1 or Hq.
 *   lse   float32 [B, Hq, Nq] contiguous, natural-log log-sum-exp per row.
 * bf16 query tiles pack heads: block_q == 128 puts 128 queries of one head in
 * a tile; block_q == 64 puts 64 queries of two heads of one key/value group in
 * a tile and needs Hm == 1 and an even Hq/Hkv. block_k is 64 or 128.
 * Rows with no visible key get out = 0 and lse = -inf. */
mfa_status mfa_fwd(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v,
                   const mfa_mask_desc* mask, const mfa_tensor* out, float* lse,
                   void* stream);

/* Additive ALiBi bias on the scores of visible pairs, from the Ascend CANN
 * "Mask Compression" page (ALiBi paragraphs): a per-head slope times a bias
 * matrix, the slopes passed in. The page's figures of the bias matrices are
 * lost; the bias of visible pair (row i, key j) is read as
 *   MFA_BIAS_ALIBI       slope_h * (j - i)       (right-aligned)
 *   MFA_BIAS_ALIBI_SQRT  -slope_h * sqrt(|i - j|)
 *   MFA_BIAS_ALIBI_LEFT  slope_h * j             (left-aligned: the output of
 *                        MFA_BIAS_ALIBI, lse larger by slope_h * i)
 * The boolean visibility still comes from the mask description. */
#define MFA_BIAS_NONE 0
#define MFA_BIAS_ALIBI 1
#define MFA_BIAS_ALIBI_SQRT 2
#define MFA_BIAS_ALIBI_LEFT 3
typedef struct mfa_bias {
  int32_t kind;           /* MFA_BIAS_*                                   */
  int32_t reserved;       /* 0                                            */
  const float* slopes;    /* DEVICE float32 [Hq], one slope per query head */
} mfa_bias;

/* mfa_fwd with an additive bias (bias != NULL; kind MFA_BIAS_NONE is plain
 * mfa_fwd). bf16 inputs only: fp32 inputs with a bias return
 * MFA_ERR_UNSUPPORTED. Every computed tile, FULL or PARTIAL, adds the bias
 * per element; the tile map is the mask's own. */
mfa_status mfa_fwd_bias(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v,
                        const mfa_mask_desc* mask, const mfa_bias* bias, const mfa_tensor* out, float* lse,
                        void* stream);

/* Size of the device array mfa_fwd_noalloc keeps its tile map and work
 * counters in: 16 MiB, held on every GPU where the library's kernels are
 * loaded, until the process exits. */
#define MFA_NOALLOC_SCRATCH_BYTES (16u << 20)

/* The forward pass for callers that cannot allocate device memory: for
 * example a plugin inside a host application that owns the GPU allocator and
 * passes in only the tensors, or code that must not allocate at this point of
 * its pipeline. The pages have no counterpart; this is a convenience of the
 * library. It does what mfa_build_tile_map followed by mfa_fwd do, but the
 * tile map (block_q x block_k, each 64 or 128) and the forward pass's work
 * counters live in a fixed array of MFA_NOALLOC_SCRATCH_BYTES that the library
 * itself holds in device memory; nothing is allocated by anyone. mask->map is
 * ignored. q, k, v, out and lse are as for mfa_fwd.
 * - Every argument is checked on the host first, as mfa_fwd checks it; a map
 *   larger than MFA_NOALLOC_SCRATCH_BYTES (mfa_tile_map_bytes) returns
 *   MFA_ERR_UNSUPPORTED. A rejected call launches nothing and leaves the
 *   array as it was.
 * - dev_err: optional DEVICE pointer to one uint32; after the pass it receives
 *   the device error bits (MFA_DEVERR_*) by a device-to-device copy on
 *   `stream`. NULL skips the copy.
 * - The array's device address is looked up (cudaGetSymbolAddress) with the
 *   call's device current: on the first call on each device, and again on
 *   every later call made while `stream` is not capturing, so a
 *   cudaDeviceReset between calls leaves no stale address behind. Make the
 *   first call on each device before any stream capture.
 * - Every call on a device shares the one array and leaves its contents in it
 *   (each call clears and rebuilds what it uses). Calls that overlap on the
 *   GPU race: order them (one stream, or events between streams). */
mfa_status mfa_fwd_noalloc(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v,
                           const mfa_mask_desc* mask, int32_t block_q, int32_t block_k,
                           const mfa_tensor* out, float* lse, uint32_t* dev_err, void* stream);

/* Test hook for the bounded waits of the forward kernel; the pages have no
 * counterpart. Every wait of the bf16 forward pipeline gives up after a time
 * limit (2 s by default): the CTA then unwinds (its roles leave, copies already
 * issued land, TMEM is released), MFA_DEVERR_TIMEOUT is set in the map's error
 * word and that launch's outputs are invalid. Arming this hook makes the next
 * bf16 mfa_fwd / mfa_fwd_bias launch in the process use a limit of wait_us
 * microseconds and have CTA 0 withhold its first K tile (it issues no copy and
 * no arrival for it), so that one wait runs out; the hook then disarms itself.
 * Nothing faults: the wait that runs out is on a tile no copy will ever fill.
 * wait_us in [1, 1000000], else MFA_ERR_INVALID_ARG. Host only. */
mfa_status mfa_test_arm_fwd_timeout(uint32_t wait_us);

/* Bytes of the DEVICE workspace mfa_bwd needs for these shapes (0 on invalid
 * shapes). Host only. */
size_t mfa_bwd_workspace_bytes(int32_t B, int32_t Hq, int32_t Nq, int32_t Nk, int32_t D);

/* Gradients of the forward pass on `stream`, for a loss whose gradient with
 * respect to out is dout and which does not use lse. This is the derivative
 * of mfa_fwd's definition by the chain rule; the pages give no backward
 * formulas. With P = exp(S - lse) on visible pairs and 0 elsewhere:
 *   dv = P^T dout, dS = P * (dout v^T - rowsum(dout * out)),
 *   dq = dS k / sqrt(D), dk = dS^T q / sqrt(D).
 * Key/value head g receives the sums over its query heads g*G .. g*G+G-1.
 *   q, out, dout, dq  [B, Hq, Nq, D] bf16;  k, v, dk, dv  [B, Hkv, Nk, D] bf16;
 *       stride[3] == 1, other strides and base addresses 16-byte aligned.
 *       out and lse are those mfa_fwd returned for q, k, v and this mask.
 *   lse   float32 [B, Hq, Nq] contiguous.
 *   mask  description with mask->map built from it by mfa_build_tile_map
 *         (the forward pass's map serves) with block_k = 128 and block_q 64
 *         or 128; Hm must be 1. The gradient kernel walks 64-query tiles; a
 *         128-row map tile gives both of its halves its class.
 *   workspace  DEVICE buffer of at least mfa_bwd_workspace_bytes(B, Hq, Nq,
 *         Nk, D) bytes, 256-byte aligned, owned by the caller; no contents are
 *         needed on entry (it holds an fp32 dq accumulator, per-row softmax
 *         statistics and the map transposed to per-key-tile lists).
 * D must be 128. Keys that no query sees get dk = dv = 0. Four kernel
 * launches: statistics, transposed lists, the gradient kernel, dq conversion
 * (none of them allocates). A bounded wait that gives up sets
 * MFA_DEVERR_TIMEOUT in the map's error word. Calls that share a workspace
 * must not overlap on the GPU.
 * Errors: MFA_ERR_INVALID_ARG (NULL pointers, small or misaligned workspace),
 * MFA_ERR_SHAPE_MISMATCH, MFA_ERR_UNSUPPORTED (dtype other than bf16, D != 128,
 * Hm != 1, block_k != 128), MFA_ERR_CUDA. */
mfa_status mfa_bwd(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v, const mfa_tensor* out,
                   const mfa_tensor* dout, const float* lse, const mfa_mask_desc* mask, const mfa_tensor* dq,
                   const mfa_tensor* dk, const mfa_tensor* dv, void* workspace, size_t workspace_bytes,
                   void* stream);

/* Bytes of the DEVICE workspace mfa_decode needs for these sizes and n_split
 * (0 = the automatic slot partition, which depends on the current device's SM
 * count; 256 when no row is split; 0 on invalid sizes). Host only. */
size_t mfa_decode_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t Nq, int32_t D, int32_t sel_k,
                                  int32_t n_split);

/* Selected-key attention for a few query rows (decode), from the pull request
 * "vulkan : selected-key flash attention for QSA block selection" (overview
 * and kernel description), on `stream`.
 *   q, out  [B, Hq, Nq, D] bf16;  k, v  [B, Hkv, Nk, D] bf16 (the cache);
 *           D in {128, 256}, G = Hq / Hkv in {1, 2, 4, 8, 16}, G * D <= 2048;
 *           stride[3] == 1, other strides and base addresses 16-byte aligned.
 *   sel     DEVICE int32 [B, Hkv, Nq, sel_k] contiguous: for every (batch,
 *           key/value head, query row) a list of 64-key block indices, shared
 *           by the head's G query heads. -1 = no entry; a block listed twice
 *           counts once; entries outside [-1, ceil(Nk/64)) are ignored and set
 *           MFA_DEVERR_SEL. sel_k <= 256.
 *   Query row i sits at position i + Nk - Nq: it sees key j when j's block is
 *   listed and j <= i + Nk - Nq (with Nq == Nk, the rule of MFA_MASK_BLOCKSEL).
 *   Rows that see no key get out = 0 and lse = -inf.
 *   lse     float32 [B, Hq, Nq] contiguous, natural log.
 *   n_split how the lists are cut among CTAs. n_split >= 1: n_split parts of
 *           ceil(sel_k / n_split) slots per list, one CTA each. 0: the lists
 *           of all rows laid end to end and cut into equal slot ranges,
 *           about one per SM (at least 2 slots, whole lists when a range
 *           holds one or more), so a CTA may finish one row and start the
 *           next. A row met by several CTAs is merged by a second kernel
 *           (empty parts carry m = -FLT_MAX, so no exp(-inf - -inf) arises),
 *           launched as a programmatic dependent of the first; `workspace`
 *           (DEVICE, 256-byte aligned, mfa_decode_workspace_bytes bytes,
 *           owned by the caller) then holds the partial results.
 *   dev_err DEVICE uint32 the kernels OR MFA_DEVERR_* bits into (required; the
 *           caller clears it).
 * Errors: MFA_ERR_INVALID_ARG, MFA_ERR_SHAPE_MISMATCH, MFA_ERR_UNSUPPORTED
 * (dtype, D, G, sizes, Nk == 0), MFA_ERR_CUDA. */
mfa_status mfa_decode(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v, const int32_t* sel,
                      int32_t sel_k, const mfa_tensor* out, float* lse, int32_t n_split, void* workspace,
                      size_t workspace_bytes, uint32_t* dev_err, void* stream);

/* Synchronise `stream`, read the map's error word into *err_bits (if not
 * NULL) and return MFA_ERR_DEVICE when it is non-zero, MFA_OK otherwise. */
mfa_status mfa_get_device_status(const mfa_tile_map* map, void* stream, uint32_t* err_bits);

#ifdef __cplusplus
}
#endif

#endif /* MFA_H_ */
