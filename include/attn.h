/*
 * attn.h -- C ABI of libattn_b200.so: exact, IO-aware attention on B200 (sm_100a).
 *
 * The library computes scaled dot-product attention
 *
 *     O = softmax(Q K^T * scale + mask) V        (per head; LSE written alongside)
 *
 * exactly, FlashAttention-style: Q, K and V are tiled through shared memory and
 * tensor memory with an online softmax (running row max m and sum l, with the
 * accumulator rescaled when m grows), so the N x N score matrix S and the
 * probability matrix P never reach HBM.
 *
 * Sources for what is computed:
 *   - SDPA definition: "Attention Mechanism Optimization for Efficient LLM
 *     Inference", section "Background: Scaled Dot-Product Attention".
 *   - Tiling, online softmax, exactness (Theorem 1) and block-sparse skipping:
 *     "FlashAttention: memory-saving exact attention", sections 2, 3 and 6.
 *   - GQA head grouping (contiguous groups share one KV head) and the decode
 *     step over a KV cache: the inference page, sections "Grouped-Query
 *     Attention" and "Two Phases of Inference / Decode".
 *   - Frame-aligned block-sparse masks and the removal of partial tiles:
 *     "TPU attention optimisation guide" (aibase.it), step 3.
 *
 * Conventions shared by every call
 *   - Every function returns an attn_status code; no call aborts or exits.
 *     attn_last_error_detail() gives the text of the last failure on the
 *     calling thread.
 *   - Tensors are contiguous and row-major in the layouts stated per call.
 *     Device pointers must be 16-byte aligned.  The caller owns every buffer;
 *     the library never frees or reallocates caller memory.  The library sees
 *     pointers, not sizes: the caller guarantees that every buffer holds the
 *     elements its layout states for the sizes passed (the Python binding
 *     checks this before it passes a pointer).
 *   - Streams: "stream" is a cudaStream_t passed as void* (NULL = legacy
 *     default stream).  Compute calls are asynchronous on that stream.
 *     Argument errors are returned at once, before any launch.  Errors that a
 *     kernel detects (a bounded wait that ran out, a cache length outside
 *     [0, Lmax]) are latched in a device word and returned by a later
 *     attn_sync_status().
 *   - Workspace: the library owns a per-device workspace (tile schedules,
 *     split-KV partials, backward and key-statistics scratch, error word).
 *     It grows on demand with cudaMalloc and is released by attn_shutdown().
 *     A call that must grow it synchronises the device.  Calls that use the
 *     same scratch (decode, backward; key statistics) must not run
 *     concurrently on different streams: order them.
 *   - Masks.  NONE: every key allowed.  CAUSAL: key j allowed for query i iff
 *     j <= i + (Nkv - Nq) (bottom-right alignment).  BLOCK: allowed iff
 *     block_map[i/16][j/16] != 0, a host uint8 array of
 *     [ceil(Nq/16)][ceil(Nkv/16)].  A row with no allowed key gets O = 0 and
 *     LSE = -inf.
 *   - LSE is ln(sum_j exp(scale * q_i . k_j)) over the allowed j, in fp32.
 *   - GQA: Hq % Hkv == 0; query head h reads KV head h / (Hq / Hkv).
 */
#ifndef EXACT_IO_AWARE_SM_B200_ATTN_H
#define EXACT_IO_AWARE_SM_B200_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_NULL = 1,            /* a required pointer is NULL */
  ATTN_ERR_SHAPE = 2,           /* a size is out of range or inconsistent */
  ATTN_ERR_ALIGN = 3,           /* a device pointer is not 16-byte aligned */
  ATTN_ERR_UNSUPPORTED = 4,     /* head dim / dtype / device not supported */
  ATTN_ERR_MASK = 5,            /* bad mask kind or missing block map */
  ATTN_ERR_CUDA = 6,            /* a CUDA runtime or driver call failed */
  ATTN_ERR_DEVICE_TIMEOUT = 7,  /* a kernel's bounded wait ran out */
  ATTN_ERR_WORKSPACE = 8,       /* workspace allocation failed */
  ATTN_ERR_DEVICE_ARG = 9       /* a kernel found a bad device-side argument (seqlens) */
} attn_status;

typedef enum { ATTN_MASK_NONE = 0, ATTN_MASK_CAUSAL = 1, ATTN_MASK_BLOCK = 2 } attn_mask_kind;

typedef enum { ATTN_BF16 = 0, ATTN_F32 = 1 } attn_dtype;

/* Block-map granularity (rows and columns). */
#define ATTN_MAP_GRAIN 16

/*
 * attn_fwd -- prefill attention over full Q, K, V.
 *
 * Passage: FlashAttention page, section 3 (the fused tiled forward pass) and
 * section 6 (block-sparse: tiles that the block mask zeroes are skipped); the
 * causal mask; GQA sharing of K/V.
 *
 *   q      device, [B, Nq, Hq, d]   (dtype)
 *   k, v   device, [B, Nkv, Hkv, d] (dtype)
 *   o      device, [B, Nq, Hq, d]   (dtype; written)
 *   lse    device, [B, Hq, Nq] fp32 (written); may be NULL to skip
 *   scale  logit scale, typically 1/sqrt(d)
 *   mask_kind  attn_mask_kind
 *   block_map  host uint8 [ceil(Nq/16)][ceil(Nkv/16)] for ATTN_MASK_BLOCK,
 *              ignored (may be NULL) otherwise.  Read during the call only.
 *   dtype  ATTN_BF16: tensor-core path (tcgen05, fp32 accumulation, P rounded
 *          to bf16 for the PV product).  d in {64, 128}.
 *          ATTN_F32: fp32 inputs and output, exact fp32 CUDA-core path for
 *          small problems.  d in {32, 64, 128}.
 * Limits: B, Hq, Hkv >= 1; Nq, Nkv >= 1; B*Hq*ceil(Nq/16) < 2^31.
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED, MASK, CUDA, WORKSPACE.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int Nq, int Nkv, int d, float scale, int mask_kind, const uint8_t* block_map,
             int dtype, void* stream);

/*
 * attn_decode -- single-token decode over a KV cache (split-KV + LSE combine).
 *
 * Passage: the inference page, section "Decode" (the new query attends to
 * every cached key/value) and section "Why Decode is Memory-bound"; the
 * combine uses the block merge rule of the FlashAttention page, section 2.
 *
 *   q         device, [B, Hq, d] bf16 (the newest token's query per sequence)
 *   k_cache   device, [B, Lmax, Hkv, d] bf16
 *   v_cache   device, [B, Lmax, Hkv, d] bf16
 *   seqlens   device, int32 [B]; sequence b attends to cache rows
 *             0 .. seqlens[b]-1.  Rows at or above seqlens[b] never affect
 *             the result, whatever they hold (NaN included); the kernel may
 *             read up to 15 of them, never at or beyond Lmax.
 *             A value outside [0, Lmax] latches ATTN_ERR_DEVICE_ARG and that
 *             sequence gets O = 0, LSE = -inf; 0 gives O = 0, LSE = -inf.
 *   o         device, [B, Hq, d] bf16 (written)
 *   lse       device, [B, Hq] fp32 (written); may be NULL
 * Limits: d == 128 or 64; 1 <= Lmax; Hq / Hkv <= 8.
 * Scratch: fp32 partials in the library workspace, B*Hq*ceil(Lmax/chunk)*(d+1)
 * floats (chunk = 512 keys).
 */
int attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                void* o, float* lse, int B, int Hq, int Hkv, int Lmax, int d, float scale,
                void* stream);

/*
 * attn_decode_multi -- decode of the Sq newest tokens of each sequence at
 * once (several tokens per step, e.g. multi-token prediction), over the same
 * KV cache read once for all of them.
 *
 * Passage: as attn_decode; the tokens' own K/V rows are already in the cache
 * (positions seqlens[b]-Sq .. seqlens[b]-1), and token s (0-based) attends to
 * rows 0 .. seqlens[b]-Sq+s: the last Sq rows of a causal prefill with
 * Nq = Sq and Nkv = seqlens[b] (bottom-right aligned causal mask).
 *
 *   q         device, [B, Sq, Hq, d] bf16
 *   k_cache, v_cache, seqlens   as attn_decode
 *   o         device, [B, Sq, Hq, d] bf16 (written)
 *   lse       device, [B, Hq, Sq] fp32 (written); may be NULL
 * A token that sees no row (seqlens[b] - Sq + s < 0) gets O = 0, LSE = -inf.
 * Limits: as attn_decode, and (Hq / Hkv) * Sq <= 16 (the query heads of a KV
 * group times the tokens fill one or two 8-column MMA operands that share
 * every K/V fragment), else ATTN_ERR_UNSUPPORTED.  Sq = 1 is attn_decode.
 * Scratch: B*Sq*Hq*ceil(Lmax/512)*(d+1) floats of library workspace.
 */
int attn_decode_multi(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                      void* o, float* lse, int B, int Sq, int Hq, int Hkv, int Lmax, int d, float scale,
                      void* stream);

/*
 * attn_frame_block_map -- block map of the frame-aligned video mask.
 *
 * Passage: TPU attention guide, step 3 (the mask's live region follows frame
 * boundaries; each query frame attends to its own frame, the previous frame
 * and the reference frame 0).  Query frame f sees key frames {0, f-1, f}.
 *   out  host, uint8 [nb][nb], nb = ceil(n_frames*frame_len/16)
 * Requires frame_len % 16 == 0 (so that no 16x16 block straddles frames);
 * else ATTN_ERR_SHAPE.
 */
int attn_frame_block_map(int n_frames, int frame_len, uint8_t* out);

/*
 * attn_classify -- full / empty / partial class of every tile of a grid.
 *
 * Passage: TPU attention guide, step 3 (measure the share of partial blocks
 * among live blocks; find a tile size that splits the mask into tiles fully
 * inside or outside it).
 *   out  host, uint8 [ceil(Nq/tq)][ceil(Nkv/tk)]: 0 empty, 1 full, 2 partial.
 *        Edge tiles are classified by their elements inside [0,Nq) x [0,Nkv).
 */
int attn_classify(int mask_kind, const uint8_t* block_map, int Nq, int Nkv, int tq, int tk,
                  uint8_t* out);

/*
 * attn_plan -- the tile schedule attn_fwd would run for a mask (host only).
 *
 * Q tiles hold at most 128 rows and never mix rows with different block-map
 * rows, so under a BLOCK mask every KV tile is full (no predicate); under a
 * CAUSAL mask the diagonal tiles are partial; a KV tile that runs past Nkv is
 * partial.  Empty tiles are never listed.
 *   qtiles   host int32 [qcap][4]: (row0, nrows, first_kv, n_kv), or NULL
 *   kvtiles  host int32 [kvcap][3]: (col0, ncols, partial), or NULL
 *            ncols is a multiple of 16 and at most 128.
 *   *n_q, *n_kv  receive the counts (always written).
 * Returns ATTN_ERR_SHAPE if a capacity is too small (counts still written).
 */
int attn_plan(int mask_kind, const uint8_t* block_map, int Nq, int Nkv, int32_t* qtiles, int qcap,
              int32_t* kvtiles, int kvcap, int* n_q, int* n_kv);

/*
 * attn_sync_status -- synchronise `stream` and return (and clear) the error
 * word latched by kernels on the current device (ATTN_OK if none).
 */
int attn_sync_status(void* stream);

/* Copy the text of the last failure on this thread into buf (NUL-terminated). */
int attn_last_error_detail(char* buf, int len);

/* Release every workspace the library holds (all devices).  Idempotent. */
int attn_shutdown(void);

/* Size of the fixed device array that attn_decode_noalloc uses as scratch. */
#define ATTN_NOALLOC_SCRATCH_BYTES (32u << 20) /* 32 MiB */

/*
 * attn_decode_noalloc -- attn_decode for callers that cannot allocate.
 *
 * The source pages have no counterpart for this entry point.
 *
 * Some callers cannot let a library call cudaMalloc: a host framework that
 * owns all device memory through its own pool, a serving process whose memory
 * budget is fixed at start-up, or a caller that cannot take the device-wide
 * synchronisation cudaMalloc / cudaFree may cause.  This variant computes the
 * same decode as attn_decode (same arguments, layouts and kernels) but keeps
 * its scratch (the per-split fp32 partials and an error word) in one fixed
 * file-scope device array of ATTN_NOALLOC_SCRATCH_BYTES.  Every GPU that loads
 * the library holds that array until the process exits.  The call itself
 * performs no cudaMalloc, cudaFree or other allocating call.
 *
 *   Scratch needed: 256 + 4 * B*Hq*ceil(Lmax/512)*(d+1) bytes; a shape that
 *   needs more than ATTN_NOALLOC_SCRATCH_BYTES returns ATTN_ERR_WORKSPACE
 *   (attn_last_error_detail says how much it needed), before any GPU work.
 *   Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it; make that
 *   first call before any stream capture.  attn_shutdown forgets the cached
 *   addresses: call it before a cudaDeviceReset, so that the next call looks
 *   the array up again in the new context.
 *   Sharing: every call on a device uses the same array, and the array keeps
 *   the previous call's contents (each call writes every partial it reads).
 *   Calls that overlap on the GPU (different streams, or other host threads)
 *   race on the array: order them.
 *   Errors: as attn_decode for arguments (a device that is not sm_100 gives
 *   ATTN_ERR_UNSUPPORTED).  Errors found on the device go to an error word
 *   inside the array, not to the one attn_sync_status reads: a seqlens entry
 *   outside [0, Lmax] (that sequence gets O = 0 and LSE = -inf) and a bounded
 *   wait that ran out (O and LSE of that call are then undefined).  The word
 *   stays latched until attn_decode_noalloc_status reads and clears it.
 */
int attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* seqlens, void* o, float* lse, int B, int Hq, int Hkv,
                        int Lmax, int d, float scale, void* stream);

/*
 * attn_decode_noalloc_status -- synchronise `stream`, then return (and clear)
 * the error word of attn_decode_noalloc on the current device: ATTN_OK,
 * ATTN_ERR_DEVICE_TIMEOUT or ATTN_ERR_DEVICE_ARG (see above).  Allocates
 * nothing.  The source pages have no counterpart for it either.
 */
int attn_decode_noalloc_status(void* stream);

/*
 * attn_bwd -- gradients of attn_fwd (bf16) for an upstream gradient dO.
 *
 * Passage: "FlashAttention: memory-saving exact attention", section 4: the
 * backward keeps only O and the row statistics of the forward and recomputes
 * S and P from Q, K and those statistics, block by block, in on-chip memory.
 * With P = exp(S - LSE), D_i = rowsum(dO_i * O_i):
 *   dV = P^T dO,  dS = P * (dO V^T - D),  dQ = scale dS K,  dK = scale dS^T Q,
 * dK and dV of a KV head summing over its Hq/Hkv query heads.
 *
 *   q, o, dout  device, [B, Nq, Hq, d] bf16 (o: the forward output)
 *   k, v        device, [B, Nkv, Hkv, d] bf16
 *   lse         device, [B, Hq, Nq] fp32, the forward LSE (natural log)
 *   dq          device, [B, Nq, Hq, d] bf16 (written)
 *   dk, dv      device, [B, Nkv, Hkv, d] bf16 (written)
 *   mask_kind, block_map  as attn_fwd (NONE, CAUSAL or BLOCK with its host map)
 * Limits: d == 64 or 128; all pointers 16-byte aligned.
 * Scratch: 2*B*Hq*ceil(Nq/128)*128 floats of library workspace.
 * Under a BLOCK mask the live 128 x 128 tile pairs are listed on the host
 * (cached per map, like attn_fwd's schedules) with the bitmap of their 16 x 16
 * blocks; only live pairs are computed.
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED (d), MASK, CUDA, WORKSPACE;
 * a bounded wait that runs out latches ATTN_ERR_DEVICE_TIMEOUT.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
             void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nkv, int d, float scale,
             int mask_kind, const uint8_t* block_map, void* stream);

/*
 * attn_debug_fault -- test hook for the device time-out path.
 *
 * kind 1: the next bf16 attn_fwd call on this thread makes CTA 0 skip its
 * first K tile load, so a bounded wait in that CTA runs out (about 2 s);
 * the kernel then stops cleanly, the context stays usable, and the next
 * attn_sync_status() returns ATTN_ERR_DEVICE_TIMEOUT.  The outputs of that
 * call are undefined.  kind 0 clears a pending fault.  Nothing else uses it.
 */
int attn_debug_fault(int kind);

/* Library version string, e.g. "exact_io_aware_sm_b200 0.1". */
const char* attn_version(void);

/*
 * attn_key_stats -- key statistics for the bound-based softmax.
 *
 * Passage: "TPU attention optimisation guide: collective overlap and mask
 * removal, verified by trace", step 4: centring the keys on their mean leaves
 * the softmax unchanged and tightens the Cauchy-Schwarz bound of the scores.
 *
 *   k       device, [B, Nkv, Hkv, d] bf16
 *   kbar    device, fp32 [B, Hkv, d] (written): mean of the Nkv keys of each
 *           (b, KV head)
 *   radius  device, fp32 [B, Hkv] (written): max_j ||k_j - kbar||
 * Limits: d == 64 or 128; B*Nkv*Hkv < 2^31; k and kbar 16-byte aligned,
 * radius 4-byte aligned.
 * Scratch: B*Hkv*ceil(Nkv/128)*d floats of library workspace.
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED, CUDA, WORKSPACE.
 */
int attn_key_stats(const void* k, float* kbar, float* radius, int B, int Nkv, int Hkv, int d, void* stream);

/*
 * attn_fwd_bound -- attn_fwd (bf16) with the bound-based softmax.
 *
 * Passage: the TPU guide, step 4: each row's running max is replaced by an
 * upper bound of its scores, scale*(q.kbar + ||q||*radius) (Cauchy-Schwarz on
 * the centred keys), so no row max is taken and nothing is rescaled; a row
 * whose bound could push a probability below 2^-100 (2*scale*log2(e)*
 * ||q||*radius > 100) falls back to the running max.  The guide checks this
 * per head; here it is checked per row (a head qualifies iff all its rows do).
 * O and LSE are those of attn_fwd up to rounding.
 *
 *   q, k, v, o, lse, sizes, scale, mask_kind, block_map: as attn_fwd
 *   kbar, radius  device, from attn_key_stats on the same k
 *   n_fallback    device int32 (may be NULL): the number of rows that kept
 *                 the running max is added to it
 * Limits: d == 64 or 128; as attn_fwd otherwise.
 * Errors: as attn_fwd.
 */
int attn_fwd_bound(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                   int Nkv, int d, float scale, int mask_kind, const uint8_t* block_map, const float* kbar,
                   const float* radius, int* n_fallback, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_IO_AWARE_SM_B200_ATTN_H */
