/*
 * axis_attn.h -- C ABI of the B200 (sm_100a) fused causal GQA softmax attention.
 *
 * The operation (forward and backward of scaled-dot-product softmax attention,
 * causal mask optional, GQA head sharing, bf16 storage with fp32 accumulation,
 * attention probabilities never written to device memory) is the fused flash
 * attention of the "Axis" page (zyoralabs.com/axis, feature list: "fused flash
 * attention, forward and backward"; "bf16 storage ... fp32 accumulation"), with
 * KV groups from the same page's second code sample (n_heads / n_kv_heads) and
 * the [B, S, H, D] tensor layout of the axiomlm page (PyPI, Quick Start section
 * 8).  The pages give no formula; the library computes, for batch b, query head
 * h, kv head kv = h / (Hq / Hkv), and query row i:
 *
 *   s_ij = scale * <Q[b,i,h,:], K[b,j,kv,:]>,  visible iff (!causal || j <= i)
 *   LSE[b,h,i] = ln sum_{visible j} exp(s_ij)         (natural log, fp32)
 *   P_ij = exp(s_ij - LSE[b,h,i]),  O[b,i,h,:] = sum_j P_ij V[b,j,kv,:]
 *
 * and the analytic gradients dQ, dK, dV of sum(dO * O), with dK and dV summed
 * over the query heads of each kv group.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors: q, o, dO, dq are [B, S, Hq, D]; k, v, dk, dv are [B, S, Hkv, D];
 *    all bf16, contiguous, row-major.  lse is fp32 [B, Hq, S].
 *  - Pointers are DEVICE pointers owned by the caller and must be 16-byte
 *    aligned.  The library allocates no device memory and keeps no pointer
 *    after a call returns, apart from the fixed scratch array of
 *    axis_attn_bwd_noalloc() (below), which is part of the library's image
 *    and whose device address it looks up once per device.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *    is the legacy default stream), perform no host synchronisation and may be
 *    captured in a CUDA graph.
 *  - Requirements: B, Hq, Hkv, S >= 1; Hq % Hkv == 0; D in {64, 128};
 *    scale finite and > 0; B*S*max(Hq,Hkv)*D < 2^31; the current device is
 *    compute capability 10.0 (B200, sm_100a).
 *  - Errors: a violated requirement returns a non-zero axis_attn_status before
 *    anything is launched, and the outputs are left untouched.  A launch or
 *    driver failure returns AXIS_ATTN_ERR_CUDA.  A device-side wait that runs
 *    past its time limit (which signals a bug, never expected in use) makes the
 *    kernel stop early, release its resources and set a device status word
 *    that axis_attn_get_status() reports as AXIS_ATTN_ERR_TIMEOUT.
 */
#ifndef AXIS_ATTN_H
#define AXIS_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    AXIS_ATTN_OK = 0,
    AXIS_ATTN_ERR_NULL = 1,        /* a required pointer is NULL */
    AXIS_ATTN_ERR_ALIGN = 2,       /* a pointer is not 16-byte aligned */
    AXIS_ATTN_ERR_SHAPE = 3,       /* a size, head ratio or scale is invalid */
    AXIS_ATTN_ERR_UNSUPPORTED = 4, /* D not in {64,128}, or not a CC 10.0 device */
    AXIS_ATTN_ERR_WORKSPACE = 5,   /* workspace NULL, misaligned or too small */
    AXIS_ATTN_ERR_CUDA = 6,        /* a CUDA runtime/driver call failed */
    AXIS_ATTN_ERR_TIMEOUT = 7,     /* a device-side wait ran out (see above) */
    AXIS_ATTN_ERR_INDEX = 8        /* a device-side index (decode page table, length) was out of range */
} axis_attn_status;

/*
 * Forward.  Writes o [B,S,Hq,D] (bf16) and lse [B,Hq,S] (fp32, natural log,
 * scale included: lse = ln sum_j exp(scale * q.k_j) over visible keys).
 * causal != 0 applies the mask j <= i (one sequence length for queries and
 * keys, so the diagonal is included and no row is fully masked).
 */
int axis_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                  int B, int Hq, int Hkv, int S, int D, float scale, int causal,
                  void* stream);

/*
 * Bytes of device workspace axis_attn_bwd() needs for these sizes (0 if the
 * sizes are invalid).  It holds, per (b, query head), fp32 rows of
 * log2-scaled LSE and of Dr = rowsum(dO * O), padded to a multiple of 128,
 * and an fp32 dQ accumulator [B, Hq, S, D]; each section starts on a 256-byte
 * boundary.  Small problems add two fp32 sections [hsplit, B, S, Hkv, D] of
 * partial dK, dV (see axis_attn_bwd_head_split()).
 */
size_t axis_attn_bwd_workspace_bytes(int B, int Hq, int Hkv, int S, int D);

/*
 * How many CTAs share each (b, kv head, 128-key tile) of the backward main
 * kernel: 1, or for small problems -- fewer than 148 such tiles and more
 * than one query head per kv head -- the smallest divisor of G = Hq / Hkv
 * that gives at least 148 CTAs (else G).  The G query heads of a kv head are
 * then dealt over that many CTAs, each writes its fp32 share of dK and dV to
 * the workspace, and one more kernel adds the shares up in a fixed order
 * into dk and dv (so the result stays bitwise reproducible).  0 for invalid
 * sizes.  Informational: the other calls apply it themselves.
 */
int axis_attn_bwd_head_split(int B, int Hq, int Hkv, int S, int D);

/*
 * Backward.  Given the forward's inputs q, k, v, its outputs o and lse, and the
 * incoming gradient dO [B,S,Hq,D], writes dq [B,S,Hq,D], dk and dv
 * [B,S,Hkv,D] (bf16; fully overwritten, not accumulated into).  dk and dv sum
 * the contributions of all Hq/Hkv query heads of a kv group.  `workspace` is a
 * caller-owned device buffer of at least axis_attn_bwd_workspace_bytes() bytes,
 * 256-byte aligned; its contents on entry do not matter and on return are
 * unspecified.  Two calls that overlap on the device must not share it.
 * dq is accumulated in fp32 by TMA reduce-add copies (cp.reduce.async.bulk,
 * one 32 KB tile per key tile) applied in arrival order, so its low-order bits
 * may vary from run to run; dk and dv do not (see axis_attn_bwd_det()).
 */
int axis_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                  const void* dO, const float* lse, void* dq, void* dk, void* dv,
                  int B, int Hq, int Hkv, int S, int D, float scale, int causal,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * The three stages axis_attn_bwd() runs, in order, on one stream, exposed so a
 * caller can overlap or time them separately.  Arguments mean what they mean
 * for axis_attn_bwd() and are validated the same way; the workspace carries the
 * state from one stage to the next, so all three must get the same workspace
 * and sizes, in this order, with nothing writing the workspace in between.
 *   prepare:  scale * Dr = scale * rowsum(dO * O) and LSE * log2(e) into the
 *             workspace (the main stage forms dS already multiplied by scale,
 *             so prepare and main must get the same scale); zeroes the fp32 dQ
 *             accumulator.  Reads o, dO, lse.
 *   main:     dk, dv (written) and the dQ accumulator (added into).  Reads q, k,
 *             v, dO and the workspace.  (With a head split, a second kernel
 *             adds up the partial dK, dV.)
 *   finalize: dq = bf16(dQ accumulator).
 */
int axis_attn_bwd_prepare(const void* o, const void* dO, const float* lse, int B, int Hq, int Hkv,
                          int S, int D, float scale, void* workspace, size_t workspace_bytes,
                          void* stream);
int axis_attn_bwd_main(const void* q, const void* k, const void* v, const void* dO, void* dk,
                       void* dv, int B, int Hq, int Hkv, int S, int D, float scale, int causal,
                       void* workspace, size_t workspace_bytes, void* stream);
int axis_attn_bwd_finalize(void* dq, int B, int Hq, int Hkv, int S, int D, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * Deterministic backward: the gradients of axis_attn_bwd(), bitwise the same
 * from run to run on the same device and inputs.  The Axis page
 * (zyoralabs.com/axis, list of published checks) reports multi-GPU weights
 * bit-identical to replicated data parallel, and the axis repository page
 * (its table of claims, "The run can be reproduced") ties reproducibility to
 * the training step; with the ordinary backward, dQ is the one output whose
 * fp32 additions happen in a run-dependent order.
 *
 * How: the main kernel computes dK and dV only (they take no cross-CTA
 * additions in either mode), and a separate pass recomputes, per 128-row
 * query tile, S = Q K^T, P and dS = P (dO V^T - Dr) for every key tile the
 * rows see and accumulates dQ = scale * sum_j dS_j K_j on chip in the fixed
 * order of the key tiles.  The extra cost is two more MMAs per tile (S and dP
 * are formed twice); the workspace holds only the per-row LSE and Dr, so
 * memory stays flat as the sequence grows (the Axis page, feature list).
 * Results agree with axis_attn_bwd() to rounding (the same products, summed
 * in another order); dk and dv are bitwise the same as axis_attn_bwd()'s.
 *
 * Arguments, layouts, ownership and errors as for axis_attn_bwd(), with the
 * smaller workspace
 *   axis_attn_bwd_det_workspace_bytes() = 2 * round256(4 * B * Hq * S_pad),
 *   S_pad = ceil(S / 128) * 128
 * (about 2.1 MB for B=4, Hq=32, S=2048), plus, with a head split
 * (axis_attn_bwd_head_split() = n > 1), 2 * round256(4 * n * B * S * Hkv * D)
 * for the partial dK, dV.  A workspace shorter than that
 * returns AXIS_ATTN_ERR_WORKSPACE and launches nothing.  Returns 0 from the
 * size function for invalid sizes.
 */
size_t axis_attn_bwd_det_workspace_bytes(int B, int Hq, int Hkv, int S, int D);
int axis_attn_bwd_det(const void* q, const void* k, const void* v, const void* o, const void* dO,
                      const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int S,
                      int D, float scale, int causal, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * Backward for callers that cannot allocate device memory: same arguments,
 * results and errors as axis_attn_bwd(), minus the workspace.  (No counterpart
 * on the pages: this is a packaging variant of the backward, not a different
 * computation.)
 *
 * Who needs it: code that runs where cudaMalloc is off limits -- inside a
 * custom allocator or memory-pool callback, in a process whose device memory
 * is fully reserved up front by a framework, or in a host path that must never
 * block on the allocator -- and cannot be handed a workspace by its caller.
 * Instead of a caller-owned workspace, the scratch lives in a fixed array built
 * into this library (AXIS_ATTN_NOALLOC_SCRATCH_BYTES = 32 MiB, 256-byte aligned)
 * that every GPU which loads the library holds until the process exits.
 *
 * Limit: the sizes must satisfy
 *   axis_attn_bwd_workspace_bytes(B, Hq, Hkv, S, D) <= 32 MiB
 * (e.g. B=2, Hq=12, S=1024, D=64 fits; B=4, Hq=32, S=2048, D=64 does not);
 * larger sizes return AXIS_ATTN_ERR_WORKSPACE and launch nothing.
 * The first call on a device looks up that device's address of the array
 * (cudaGetSymbolAddress); make that first call before capturing a stream.
 * The array is shared by every call on a device and keeps the last call's
 * contents; each call re-initialises what it reads (including zeroing its dQ
 * accumulator), but two calls that overlap on the GPU (different streams, or
 * concurrent host threads) race on it and must be serialised by the caller.
 */
#define AXIS_ATTN_NOALLOC_SCRATCH_BYTES (32u << 20)
int axis_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                          const void* dO, const float* lse, void* dq, void* dk, void* dv,
                          int B, int Hq, int Hkv, int S, int D, float scale, int causal,
                          void* stream);

/*
 * Rotary position embedding (RoPE) of Q and K, fused with the attention.  The
 * axiomlm page (PyPI) lists RoPE among its Key Features, and its Quick Start
 * (section 8) computes precompute_rope_frequencies(dim, end) and then
 * apply_rope(q, k, freqs_cis) before attention; it gives no formula.  The
 * reading taken (the complex-pair form the name freqs_cis points to): in the
 * row at sequence position s the pair (x[2p], x[2p+1]) is turned by the angle
 * s * theta_p, theta_p = base^(-2p/D):
 *   x'[2p] = x[2p] cos - x[2p+1] sin,   x'[2p+1] = x[2p] sin + x[2p+1] cos.
 *
 * axis_attn_rope_table: cs[s * D/2 + p] = (cos, sin)(s * theta_p) as fp64
 *   pairs, [S][D/2][2] (the page's freqs_cis).  fp64 because the rotated q and
 *   k are stored in bf16: the rotation is computed in fp64 and rounded once,
 *   so the stored values are the correctly rounded rotation.
 *   Requirements: 8 <= D, D % 8 == 0, base finite and > 1, cs 16-byte aligned.
 * axis_attn_rope: y = the rotation of x (inverse != 0: the transposed rotation,
 *   which carries gradients back), x, y [B, S, H, D] bf16 (y may be x), cs
 *   from axis_attn_rope_table for at least S positions.  HBM-bound.
 * axis_attn_fwd_rope: the forward of axis_attn_fwd() on the rotated q and k:
 *   o, lse as for softmax(scale * (R q)(R k)^T) V, with q and k the caller's
 *   unrotated tensors.  It writes the rotated inputs into q_rot [B, S, Hq, D]
 *   and k_rot [B, S, Hkv, D] (bf16, caller-owned; the backward reads them):
 *   one HBM-bound pass each, then the forward kernel.  (A rotation of each Q
 *   tile in shared memory after its TMA load, by one warp per SM, was built
 *   and measured: at B=4, S=2048, Hq=32, D=64 it made the forward 3.5x
 *   slower than this pass, because every rotated pair needs a table read.)
 * axis_attn_bwd_rope: the gradients with respect to the UNROTATED q and k (and
 *   v) of that forward, from q_rot and k_rot: the backward of axis_attn_bwd()
 *   (deterministic != 0: of axis_attn_bwd_det()) on the rotated inputs, with
 *   the transposed rotation applied to dQ in the finalize step (or the
 *   deterministic dQ pass) and to dK in the main kernel's epilogue.  The
 *   workspace is that of axis_attn_bwd() (or axis_attn_bwd_det()).
 * Arguments, layouts, requirements and errors otherwise as for axis_attn_fwd()
 * and axis_attn_bwd(); cs must be 16-byte aligned and cover S positions of D.
 */
int axis_attn_rope_table(double* cs, int S, int D, double base, void* stream);
int axis_attn_rope(const void* x, void* y, const double* cs, int B, int S, int H, int D, int inverse,
                   void* stream);
int axis_attn_fwd_rope(const void* q, const void* k, const void* v, const double* cs, void* o,
                       float* lse, void* q_rot, void* k_rot, int B, int Hq, int Hkv, int S, int D,
                       float scale, int causal, void* stream);
int axis_attn_bwd_rope(const void* q_rot, const void* k_rot, const void* v, const double* cs,
                       const void* o, const void* dO, const float* lse, void* dq, void* dk,
                       void* dv, int B, int Hq, int Hkv, int S, int D, float scale, int causal,
                       int deterministic, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode step against a paged KV cache: for each sequence b, the new token's
 * query row attends to every key cached for b (itself included, so no mask is
 * needed).  This is the per-token step of the axiomlm inference engine
 * (axiomlm page, PyPI: Key Features, "State-cached Key-Value (KV) decode
 * engine achieving O(1) step latency"; Quick Start section 4, "the Paged
 * KV-Cache engine"), with its GQA heads (Key Features, "4-head Grouped-Query
 * Attention").  For query head h (kv head h / (Hq / Hkv)):
 *   o[b,h,:] = sum_j P_j V_j,  P = softmax_j(scale * <q[b,h,:], K_j>),  j < seq_lens[b]
 *   lse[b,h] = ln sum_j exp(scale * <q[b,h,:], K_j>)
 *
 *  - q, o: [B, Hq, D] bf16 (one row per sequence); lse: [B, Hq] fp32.
 *  - k_cache, v_cache: [num_pages, page_size, Hkv, D] bf16, a pool of pages.
 *    Position j of sequence b is row j % page_size of page
 *    block_table[b * max_pages + j / page_size].
 *  - block_table: [B, max_pages] int32; seq_lens: [B] int32, the number of
 *    cached tokens of each sequence including the new one.  Both are DEVICE
 *    arrays read by the kernel: an entry outside [0, num_pages) that a
 *    sequence's length reaches, or a length outside [1, max_pages*page_size],
 *    is never used for a memory access; the affected keys are left out and
 *    axis_attn_get_status() reports AXIS_ATTN_ERR_INDEX.
 *  - Requirements: D in {64, 128}; Hq / Hkv <= 8; page_size a power of two in
 *    [8, 256]; B, max_pages, num_pages >= 1; scale finite and > 0; 16-byte
 *    aligned q, caches, o, lse; 4-byte aligned block_table, seq_lens.
 *  - workspace: axis_attn_decode_workspace_bytes() bytes (0 is possible:
 *    then workspace may be NULL), 256-byte aligned, caller-owned; long
 *    sequences at small batch are split over several CTAs whose partial
 *    results meet there.  Calls that overlap on the GPU must not share it.
 *  - The kernel is HBM-bound: every cached key and value is read once.
 */
size_t axis_attn_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int page_size, int max_pages);
int axis_attn_decode(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                     const int* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int D,
                     int page_size, int max_pages, int num_pages, float scale, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * The same decode step on a head-major pool: k_cache, v_cache are
 * [num_pages, Hkv, page_size, D] bf16, so one kv head's rows of a page are
 * contiguous (page_size * D * 2 bytes) instead of D * 2-byte pieces at a
 * stride of Hkv * D * 2 bytes.  Position j of sequence b is row j % page_size
 * of head kv in page block_table[b * max_pages + j / page_size].  Every other
 * argument, the workspace (axis_attn_decode_workspace_bytes), the results, the
 * requirements and the error behaviour are those of axis_attn_decode.
 */
int axis_attn_decode_hnd(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                         const int* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int D,
                         int page_size, int max_pages, int num_pages, float scale, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * Decode step with q_len new tokens per sequence at once: the engine above
 * advancing several positions in one step (a chunk of a prompt appended to
 * the cache, or several proposed tokens checked together).  The new tokens are
 * the last q_len positions of their sequence, already in the cache: new token
 * t of sequence b sits at position p = seq_lens[b] - q_len + t and, under the
 * causal mask, attends to the cached keys j <= p (the earlier new tokens and
 * itself, not the later ones).  For query head h (kv head h / (Hq / Hkv)):
 *   o[b,t,h,:] = sum_{j<=p} P_j V_j,  P = softmax_j(scale * <q[b,t,h,:], K_j>)
 *   lse[b,h,t] = ln sum_{j<=p} exp(scale * <q[b,t,h,:], K_j>)
 *
 *  - q, o: [B, q_len, Hq, D] bf16; lse: [B, Hq, q_len] fp32.  q_len = 1 is
 *    axis_attn_decode (head_major = 0) / axis_attn_decode_hnd (head_major = 1).
 *  - k_cache, v_cache: [num_pages, page_size, Hkv, D] (head_major = 0) or
 *    [num_pages, Hkv, page_size, D] (head_major = 1) bf16, read through
 *    block_table as for axis_attn_decode.
 *  - seq_lens[b]: cached tokens of sequence b, the q_len new ones included; a
 *    length outside [q_len, max_pages*page_size] is clamped and reported as
 *    AXIS_ATTN_ERR_INDEX (as are out-of-range page indices).
 *  - Requirements: those of axis_attn_decode, and 1 <= q_len <= 64,
 *    q_len <= max_pages * page_size, B * q_len * Hq * D < 2^31.  The kernel
 *    takes the G * q_len (token, head) rows of a kv head in tiles of 8 (when
 *    there are at most 8) or 16, each tile streaming the kv head's keys (the
 *    tiles of a head run side by side, so the second and later reads come
 *    from L2).
 *  - workspace: axis_attn_decode_q_workspace_bytes() bytes (0 is possible),
 *    256-byte aligned, caller-owned; calls that overlap must not share it.
 */
size_t axis_attn_decode_q_workspace_bytes(int B, int q_len, int Hq, int Hkv, int D, int page_size,
                                          int max_pages);
int axis_attn_decode_q(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                       const int* seq_lens, void* o, float* lse, int B, int q_len, int Hq, int Hkv, int D,
                       int page_size, int max_pages, int num_pages, float scale, int head_major,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronises `stream`, then returns AXIS_ATTN_ERR_TIMEOUT if any kernel of
 * this library on the current device has reported a timed-out device wait since
 * the last call, else AXIS_ATTN_ERR_INDEX if a decode step met an out-of-range
 * device-side index (and clears those reports), AXIS_ATTN_ERR_CUDA if the CUDA
 * context holds an error, else AXIS_ATTN_OK.  For tests and debugging: it
 * blocks the host.  A launch that timed out leaves its outputs undefined; it
 * does not affect later launches, whether or not this function is called in
 * between (each launch only reacts to timeouts of its own CTAs).
 */
int axis_attn_get_status(void* stream);

/*
 * Diagnostics: the raw device status word that the last axis_attn_get_status()
 * call read before clearing it (0 if none was set).  Bit 0: a wait timed out;
 * bit 1: a decode index was out of range; bits 8..15: the wait site that first
 * timed out (1..12: forward kernel, 21..32: backward main kernel, 41..42:
 * decode kernel).
 */
unsigned int axis_attn_last_status_word(void);

/* Static, human-readable text for a status code. */
const char* axis_attn_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* AXIS_ATTN_H */
