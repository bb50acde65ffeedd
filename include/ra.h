/*
 * ra.h - exact blockwise (ring) attention on one NVIDIA B200 (sm_100a).
 *
 * C ABI of libra_b200.so.  Plain pointers and sizes only; every pointer named
 * "device" is a CUDA device address, every buffer is owned by the caller, and
 * the library allocates no memory.  Calls are asynchronous on `stream`
 * (a cudaStream_t passed as void*; NULL = the legacy default stream).  Argument
 * validation is synchronous: an invalid call returns an error status before
 * anything is launched and leaves every buffer untouched.  Errors that only a
 * kernel can see (a bounded wait that ran out, an index out of range) are
 * recorded in a device status word that ra_get_device_status() reads.
 *
 * Sources, by page title and section:
 *  [TR]  TokenRing review (pith.science, arXiv 2412.20501).
 *        "What carries the argument": the update rule that stitches partial
 *        outputs, out <- out - sigma(block_lse - lse) * (out - block_out),
 *        lse <- lse - ln sigma(lse - block_lse).
 *        "Core claim" / "Referee Report, Summary": Q, K, V split along the
 *        token dimension; a flash-attention kernel returns (block_out,
 *        block_lse) per query block and key/value block.
 *        "If this is right": zigzag causal partition; grouped-query attention.
 *        "major comments, Algorithm 1 (section 3.2)": TokenRing step index.
 *  [RA]  Anthology of the SOTA, SOTA-181 (Liu et al. 2023, ring attention):
 *        each device keeps its query block and passes key/value blocks
 *        around the ring; exact attention.
 *
 * Layouts (token-major, row-major, no padding):
 *   q, out      [B, S, Hq,  D]     k, v   [B, S, Hkv, D]     lse [B, S, Hq]
 * with Hq = Hkv * gqa_groups; query head h reads KV head h / gqa_groups.
 * The softmax scale is 1/sqrt(D); lse is a natural logarithm.
 * Supported: D in {64, 128}; bf16 attention inputs (fp32 inputs to
 * ra_ring_attention are rounded to bf16, round-to-nearest-even, on entry).
 * All device pointers must be 16-byte aligned.
 */
#ifndef RA_B200_H
#define RA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RA_OK = 0,
  RA_ERR_INVALID_ARG = 1,   /* bad shape, null or misaligned pointer, bad enum  */
  RA_ERR_UNSUPPORTED = 2,   /* valid but outside what this build implements      */
  RA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than the query says  */
  RA_ERR_CUDA = 4,          /* a CUDA runtime / driver call failed               */
  RA_ERR_TIMEOUT = 5,       /* device: a bounded wait ran out (kernel returned)  */
  RA_ERR_DEVICE_BOUNDS = 6  /* device: an index check failed (access skipped)    */
} ra_status;

typedef enum { RA_F32 = 0, RA_BF16 = 1 } ra_dtype;

/* [TR] "If this is right" (zigzag) and "Referee Report, Summary" (contiguous).
 * Contiguous: block r = tokens [r*L, (r+1)*L), L = S / n_blocks.
 * Zigzag: chunk size c = S / (2 n_blocks); block r = chunk r then chunk
 * 2 n_blocks - 1 - r.  Requires S % (2 n_blocks) == 0. */
typedef enum { RA_PART_CONTIGUOUS = 0, RA_PART_ZIGZAG = 1 } ra_partition;

/* Order in which each query block meets the KV blocks.
 * Ring [RA]: at step s = 0..n-1 query block r meets KV block (r - s) mod n.
 * TokenRing [TR, Algorithm 1]: at step = 1..n KV block j meets query block
 * (j - step + 1) mod n.  The result is the same up to rounding. */
typedef enum { RA_ORDER_RING = 0, RA_ORDER_TOKENRING = 1 } ra_order;

/* How ra_ring_attention runs the schedule on one GPU.
 *  UNFUSED:          per ring step one ra_block_attn-style launch over all n
 *                    (q block, kv block) pairs of the step, writing fp32
 *                    partials, then one merge launch (ra_merge_partial).
 *  EPILOGUE_FUSED:   the same launches, the attention epilogue applies the
 *                    merge rule to the running (out, lse) in HBM itself.
 *  PERSISTENT:       one launch; each CTA owns a (query tile, head) and walks
 *                    the KV blocks in schedule order, carrying the running
 *                    softmax state on chip across block boundaries; output is
 *                    written once, in original token order.
 *  AUTO:             PERSISTENT. */
typedef enum {
  RA_SCHED_AUTO = 0,
  RA_SCHED_UNFUSED = 1,
  RA_SCHED_EPILOGUE_FUSED = 2,
  RA_SCHED_PERSISTENT = 3
} ra_sched;

/* How the block-attention kernel splits work between CTAs.
 *  ROW_PAIRS: 256 query rows per CTA (two 128-row tiles sharing K/V loads).
 *  KV_SPLIT:  128 query rows per CTA; the CTA's KV tiles are halved between
 *             its two tiles and the two partials merged on chip with the rule.
 *  CLUSTER2:  row pairs, with the KV tiles of each 256 rows halved between
 *             the two CTAs of a thread-block cluster; the partials are merged
 *             with the rule through distributed shared memory.
 *  AUTO:      ROW_PAIRS unless that gives fewer than two CTAs per SM, then
 *             KV_SPLIT. */
typedef enum {
  RA_TILING_AUTO = 0,
  RA_TILING_ROW_PAIRS = 1,
  RA_TILING_KV_SPLIT = 2,
  RA_TILING_CLUSTER2 = 3
} ra_tiling;

typedef struct {
  ra_order order;  /* default RA_ORDER_RING  */
  ra_sched sched;  /* default RA_SCHED_AUTO  */
  /* Optional cudaEvent_t handles (NULL = unused), recorded on `stream` right
   * before the first and right after the last block-attention launch of the
   * call, so a caller can time the attention kernels inside the full call. */
  void* attn_event_begin;
  void* attn_event_end;
  ra_tiling tiling; /* default RA_TILING_AUTO */
  /* Testing the failure path only; 0 (off) in normal use.  1: the TMA
   * producer of every block-attention CTA withholds the second K tile it
   * would load, so the tensor-core issuer's bounded wait for it expires
   * (about 1 s of SM clocks): the kernel records RA_ERR_TIMEOUT in the device
   * status word, every CTA stops at its next wait, in-flight copies and
   * products are drained, and the call's outputs are undefined.  The context
   * stays usable.  2 (checked build only, see ra_debug_build): the producer
   * checks its second K tile's row as if it lay past the end of the tensor;
   * the check records RA_ERR_DEVICE_BOUNDS, the copy is skipped and the CTA
   * stops.  Other values: RA_ERR_INVALID_ARG. */
  int fault_inject;
} ra_options;

/*
 * ra_block_attn - one query block against one key/value block.
 * [TR] "What carries the argument" / "Core claim": the flash-attention kernel
 * that returns (block_out, block_lse) for one block pair.
 *
 *  q          device, bf16, [B, L, Hq, D]: the rows of query block q_block
 *             (block-local, in partition order; L = S / n_blocks).
 *  k, v       device, bf16, [B, L, Hkv, D]: the rows of KV block kv_block.
 *  in_dtype   must be RA_BF16 (else RA_ERR_UNSUPPORTED).
 *  B, S       batch and full sequence length; n_blocks blocks of L tokens.
 *  q_block, kv_block   block indices in [0, n_blocks); with `partition` they
 *             give every row's original token position, used by the mask.
 *  Hq, Hkv, D head counts (Hq % Hkv == 0) and head dim (64 or 128).
 *  causal     nonzero: key j visible to query i iff pos(j) <= pos(i).
 *  block_out  device, fp32, [B, L, Hq, D], written (softmax-normalised).
 *  block_lse  device, fp32, [B, L, Hq], written.  A row that sees no key of
 *             this block gets block_lse = -inf and block_out = 0.
 */
ra_status ra_block_attn(const void* q, const void* k, const void* v, ra_dtype in_dtype,
                        int B, int S, int n_blocks, int q_block, int kv_block,
                        int Hq, int Hkv, int D, int causal, ra_partition partition,
                        float* block_out, float* block_lse, void* stream);

/*
 * ra_block_attn_merge - one ring step on one device: the block pair's
 * partial (as ra_block_attn computes it) folded into a running (out, lse) by
 * the update rule of ra_merge_partial, inside the attention kernel's
 * epilogue (the partial never reaches HBM).
 * [RA] SOTA-181: each device keeps its query block and meets one key/value
 * block per step; [TR] "What carries the argument": the partials are stitched
 * by the update rule without recomputation.
 *  q, k, v, in_dtype, B .. partition   as in ra_block_attn.
 *  out        device, fp32, [B, L, Hq, D], read and written: the running
 *             output of query block q_block.  Start from out = 0.
 *  lse        device, fp32, [B, L, Hq], read and written: the running lse;
 *             start from lse = -inf (no block merged yet).  A row that sees
 *             no key of this KV block keeps its (out, lse).
 * Every pointer must be 16-byte aligned (else RA_ERR_INVALID_ARG).  After
 * the pairs (q_block, 0 .. n_blocks-1) have all been merged, in any order,
 * (out, lse) is the block's exact attention up to rounding.
 */
ra_status ra_block_attn_merge(const void* q, const void* k, const void* v, ra_dtype in_dtype,
                              int B, int S, int n_blocks, int q_block, int kv_block,
                              int Hq, int Hkv, int D, int causal, ra_partition partition,
                              float* out, float* lse, void* stream);

/*
 * ra_merge_partial - one application of the update rule, in place, fp32.
 * [TR] "What carries the argument":
 *     out <- out - sigma(block_lse - lse) * (out - block_out)
 *     lse <- lse - ln sigma(lse - block_lse)
 *  out, lse              device fp32 [rows, D] / [rows], read and written.
 *  block_out, block_lse  device fp32 [rows, D] / [rows], read only.
 *  rows, D               rows >= 0 (0 is a no-op), D > 0 and D % 4 == 0.
 * lse = -inf marks an empty partial: merging an empty block_lse is a no-op;
 * merging into an empty lse copies the partial.
 */
ra_status ra_merge_partial(float* out, float* lse, const float* block_out,
                           const float* block_lse, int64_t rows, int D, void* stream);

/*
 * ra_merge_partials - k partials folded into one result in a single pass
 * (the same rule applied k-1 times, left to right, on chip).
 *  outs, lses    host arrays of k device pointers: fp32 [rows, D] / [rows].
 *  out, lse      device fp32 [rows, D] / [rows], written (may alias outs[0],
 *                lses[0]).  1 <= k <= 16.
 */
ra_status ra_merge_partials(const float* const* outs, const float* const* lses, int k,
                            float* out, float* lse, int64_t rows, int D, void* stream);

/*
 * ra_ring_attention - the whole method: partition, schedule, block attention,
 * merge, and the final cast / return to original token order.
 *  q, k, v       device, in_dtype (RA_BF16 or RA_F32), original token order.
 *  B, S, Hq, D   shapes; Hkv = Hq / gqa_groups.
 *  n_blocks      ring size n >= 1, <= 16; S % n == 0 (contiguous) or
 *                S % (2n) == 0 (zigzag).
 *  causal        nonzero for causal attention over original positions.
 *  out           device, out_dtype (RA_F32 or RA_BF16; bf16 is rounded to
 *                nearest even from the fp32 result), [B, S, Hq, D].
 *  lse           device fp32 [B, S, Hq].
 *  workspace     device scratch of at least ra_ring_attention_workspace()
 *                bytes (may be NULL when that is 0), 256-byte aligned.
 *  opts          NULL for defaults.
 */
ra_status ra_ring_attention(const void* q, const void* k, const void* v, ra_dtype in_dtype,
                            int B, int S, int Hq, int D, int n_blocks, int causal,
                            ra_partition partition, int gqa_groups,
                            void* out, ra_dtype out_dtype, float* lse,
                            void* workspace, size_t workspace_bytes,
                            const ra_options* opts, void* stream);

/* Bytes of workspace ra_ring_attention needs for these arguments; 0 when
 * none is needed; (size_t)-1 when the arguments are invalid. */
size_t ra_ring_attention_workspace(int B, int S, int Hq, int D, int n_blocks, int gqa_groups,
                                   ra_partition partition, ra_dtype in_dtype,
                                   ra_dtype out_dtype, const ra_options* opts);

/*
 * ra_zigzag_permute - reorder token rows between original order and the
 * partition's block order ([TR] "If this is right", zigzag partition).
 *  src, dst      device [B, S, H, D] of elem_bytes each (2 or 4); no overlap.
 *  inverse = 0:  dst[b, p] = src[b, perm[p]]   (original -> block order)
 *  inverse = 1:  dst[b, perm[p]] = src[b, p]   (block order -> original)
 * with perm[r*L + t] = r*c + t for t < c, (2n-1-r)*c + (t - c) otherwise.
 * A pure copy: bit-exact.
 */
ra_status ra_zigzag_permute(const void* src, void* dst, int B, int S, int H, int D,
                            int elem_bytes, int n_blocks, int inverse, void* stream);

/*
 * ra_ring_attention_noalloc - ra_ring_attention without a caller workspace;
 * it allocates no memory at all.  (The pages have no counterpart: this is a
 * deployment variant of the same call.)
 *
 * For callers that cannot allocate device memory at call time: code running
 * after its framework has reserved the GPU's memory for its own pool, where a
 * cudaMalloc fails or fragments that pool, and latency-bound callers that
 * cannot accept the implicit device synchronisation of cudaMalloc/cudaFree.
 * Arguments and results are those of ra_ring_attention minus the workspace.
 * The scratch the call needs (ra_ring_attention_workspace) comes from one
 * fixed device array of ra_noalloc_scratch_bytes() bytes (64 MiB) inside
 * this library, held on every GPU that loads it until the process exits.
 *  - Calls needing more scratch than that return RA_ERR_WORKSPACE before
 *    anything runs (use ra_ring_attention with a workspace instead).  The
 *    default path (bf16 inputs, persistent schedule) needs none.
 *  - The first call on a device looks up the array's device address on the
 *    current device (cudaGetSymbolAddress); make that first call before any
 *    stream capture.  `stream` must belong to the current device.  The
 *    address is kept per device and per context: after cudaDeviceReset, or
 *    once the device's primary context has been released and created again,
 *    the next call looks it up anew (the array may then sit elsewhere).
 *  - Invalid arguments return the same status as ra_ring_attention would
 *    (RA_ERR_INVALID_ARG or RA_ERR_UNSUPPORTED), before anything runs.
 *  - Every call on a device shares the one array and it keeps the last call's
 *    contents; nothing in it needs to start at zero (every scratch byte the
 *    call reads it first writes).  Calls whose work overlaps on the GPU (on
 *    different streams, or from several host threads) race on it: order them.
 */
ra_status ra_ring_attention_noalloc(const void* q, const void* k, const void* v, ra_dtype in_dtype,
                                    int B, int S, int Hq, int D, int n_blocks, int causal,
                                    ra_partition partition, int gqa_groups,
                                    void* out, ra_dtype out_dtype, float* lse,
                                    const ra_options* opts, void* stream);

/* Size in bytes of the fixed scratch array behind ra_ring_attention_noalloc. */
size_t ra_noalloc_scratch_bytes(void);

/*
 * ra_decode_attention - decode-phase attention over a KV cache, by chunks.
 * [TR] "Reading between the lines": the decode phase as KV-cache chunking;
 * every chunk's partial (out, lse) is stitched with the update rule of
 * ra_merge_partial ("What carries the argument"), in chunk order.
 *  q          device, bf16, [B, Tq, Hq, D]: the last Tq tokens of each
 *             sequence; query token i has position Skv - Tq + i.
 *  k, v       device, bf16, [B, Skv, Hkv, D]: the cache of tokens 0..Skv-1.
 *  in_dtype   must be RA_BF16 (else RA_ERR_UNSUPPORTED).
 *  Hq, Hkv    Hq % Hkv == 0; query head h reads KV head h / (Hq / Hkv);
 *             (Hq / Hkv) * Tq <= 64 (else RA_ERR_UNSUPPORTED).  D in {64, 128}.
 *             1 <= Tq <= Skv.
 *  causal     nonzero: query token i sees keys j <= Skv - Tq + i.
 *  n_splits   chunks of the cache (0 = enough to fill the GPU); the chunk
 *             length is rounded up to 64 keys, so the count actually used is
 *             ra_decode_splits() of the same arguments.
 *  out        device, out_dtype (RA_F32 or RA_BF16, nearest even), [B, Tq, Hq, D].
 *  lse        device fp32 [B, Tq, Hq], natural log.
 *  workspace  device scratch of ra_decode_workspace() bytes, 256-byte aligned
 *             (the per-chunk partials).
 */
ra_status ra_decode_attention(const void* q, const void* k, const void* v, ra_dtype in_dtype,
                              int B, int Tq, int Skv, int Hq, int Hkv, int D, int causal,
                              int n_splits, void* out, ra_dtype out_dtype, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes of ra_decode_attention for these arguments ((size_t)-1 when
 * they are invalid). */
size_t ra_decode_workspace(int B, int Tq, int Skv, int Hq, int Hkv, int D, int n_splits);

/* Chunks ra_decode_attention uses for these arguments (-1 when invalid). */
int ra_decode_splits(int B, int Tq, int Skv, int Hq, int Hkv, int D, int n_splits);

/*
 * ra_ring_attention_backward - gradients of ra_ring_attention.
 * [RA] SOTA-181: ring attention trains models (the backward pass of exact
 * attention); [TR] "What carries the argument": the forward's lse is the
 * log-sum-exp of the whole row, so every (query block, KV block) pair's
 * share of the gradient is rebuilt from it alone, P = exp(s Q K^T - lse), and
 * the shares add up:
 *     dV = sum P^T dO,  dS = P (dO V^T - Delta),  Delta = rowsum(dO * out),
 *     dQ = s sum dS K,  dK = s sum dS^T Q,        s = 1 / sqrt(D).
 *  q, k, v       device, in_dtype (RA_BF16, or RA_F32 rounded to bf16 first,
 *                as in the forward), original token order, [B, S, Hq, D] /
 *                [B, S, Hkv, D] / [B, S, Hkv, D].
 *  out           device, out_dtype (RA_F32 or RA_BF16), [B, S, Hq, D]: the
 *                forward's output for the same arguments.
 *  lse           device fp32 [B, S, Hq]: the forward's lse (natural log).
 *  dout          device, in_dtype, [B, S, Hq, D]: gradient of the loss with
 *                respect to out.
 *  B .. gqa_groups  as in ra_ring_attention (same limits).
 *  dq            device fp32 [B, S, Hq, D], written.
 *  dk, dv        device fp32 [B, S, Hkv, D], written; a KV head's gradient
 *                sums over the query heads of its group.
 *  workspace     device scratch of ra_ring_attention_backward_workspace()
 *                bytes, 256-byte aligned (never NULL: it holds Delta).
 *  opts          NULL for defaults; `order` sets the order in which the
 *                block pairs are summed (results agree up to rounding);
 *                attn_event_begin / attn_event_end bracket the two
 *                tensor-core kernels (dK/dV, then dQ).  sched, tiling and
 *                fault_inject are ignored.
 * Every pointer must be 16-byte aligned (else RA_ERR_INVALID_ARG).  Each
 * output row is written by exactly one CTA (no atomics): the result does not
 * depend on scheduling.
 */
ra_status ra_ring_attention_backward(const void* q, const void* k, const void* v, ra_dtype in_dtype,
                                     const void* out, ra_dtype out_dtype, const float* lse, const void* dout,
                                     int B, int S, int Hq, int D, int n_blocks, int causal, ra_partition partition,
                                     int gqa_groups, float* dq, float* dk, float* dv, void* workspace,
                                     size_t workspace_bytes, const ra_options* opts, void* stream);

/* Workspace bytes of ra_ring_attention_backward ((size_t)-1 when the
 * arguments are invalid). */
size_t ra_ring_attention_backward_workspace(int B, int S, int Hq, int D, int n_blocks, int gqa_groups,
                                            ra_partition partition, ra_dtype in_dtype);

/* Reads and clears the device status word (synchronises `stream`).  Returns
 * RA_OK, RA_ERR_TIMEOUT or RA_ERR_DEVICE_BOUNDS, or RA_ERR_CUDA when the read
 * itself fails. */
ra_status ra_get_device_status(void* stream);

/* Static, human-readable name of a status code. */
const char* ra_status_string(ra_status s);

/* Library version string. */
const char* ra_version(void);

/*
 * The checked build.  libra_b200_debug.so is this library compiled with
 * -DRA_DEBUG_BOUNDS: before every run-time-indexed global access (the rows
 * and heads of TMA copies, output rows, lse and Delta entries, merge rows) and
 * every segment-table read, the kernels check the index against the extent it
 * must lie in.  A failed check records RA_ERR_DEVICE_BOUNDS in the device
 * status word (ra_get_device_status), skips the access and ends the CTA's work;
 * nothing traps.  Not part of the method on the pages: a debugging aid.
 *
 * ra_debug_build: 1 in the checked build, 0 otherwise.
 * ra_get_bounds_record: the first failed check since the last read (source
 *   line, index, limit; zeros if none, and always zeros in the release
 *   build), then clears it.  Synchronous.  record: host, 3 entries.
 */
int ra_debug_build(void);
ra_status ra_get_bounds_record(int64_t record[3]);

/*
 * Per-CTA timeline (tracing).  TokenRing's per-attention-step latencies
 * (Figure 6) were read off Nsight Systems profiles ([TR] "Referee Report",
 * major comments; "Circularity Check"); this is the same kind of view one
 * level down: where each CTA of one tensor-core kernel ran and for how long.
 * Not part of the method: a profiling aid, off by default.
 *
 *  records   device, uint64 [max_ctas][4], 8-byte aligned, owned by the
 *            caller; NULL turns the timeline off (then max_ctas is ignored).
 *  max_ctas  1 .. 2^24: CTAs with blockIdx.x < max_ctas record.
 *  kernel    which kernel records: RA_TIMELINE_ATTN_FWD (attn_fwd_kernel:
 *            every block-attention launch of ra_block_attn*, ra_ring_attention*),
 *            RA_TIMELINE_BWD_DKV or RA_TIMELINE_BWD_DQ (the two tensor-core
 *            kernels of ra_ring_attention_backward*).
 *
 * While set, every launch of that kernel writes, for its CTA i < max_ctas,
 * records[i][0..3] = start and end in ns of the GPU's global timer; the SM id
 * (low 32 bits) and the CTA's work units (high 32 bits: KV tiles walked for
 * attn_fwd_kernel and the dQ kernel, query tiles walked for the dK/dV
 * kernel); and the SM clock cycles from start to end (their ratio to the
 * duration is the clock the CTA ran at).  Each launch overwrites the
 * records of the CTAs it has; a CTA whose work ends early (an abort) may
 * leave its end word unwritten.  The setting is process-wide, applies to the
 * calls made after it on any stream and device, and is not synchronised with
 * calls running on other host threads; records must stay valid until those
 * launches have completed.  Host-only: returns RA_OK, or RA_ERR_INVALID_ARG
 * for an unknown kernel, max_ctas out of range or a misaligned pointer.
 */
typedef enum {
  RA_TIMELINE_ATTN_FWD = 0,
  RA_TIMELINE_BWD_DKV = 1,
  RA_TIMELINE_BWD_DQ = 2
} ra_timeline_kernel;

ra_status ra_set_cta_timeline(uint64_t* records, int64_t max_ctas, ra_timeline_kernel kernel);

#ifdef __cplusplus
}
#endif

#endif /* RA_B200_H */
