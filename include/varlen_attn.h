/*
 * varlen_attn.h — C ABI of the B200 (sm_100a) packed variable-length
 * attention forward pass.
 *
 * The operation is VarLenAttentionOps::varlen_attention_fwd of boostr 0.2.0
 * (src/ops/traits/attention/varlen_attention.rs), "Layout contract":
 *   q   [total_q, num_heads,    head_dim]  bf16, packed queries
 *   k   [total_k, num_kv_heads, head_dim]  bf16, packed keys
 *   v   [total_k, num_kv_heads, head_dim]  bf16, packed values
 *   cu_seqlens_q / cu_seqlens_k  int32 [batch + 1], "Cumulative sequence
 *       lengths": cu[0] = 0, cu[i] = sum of the first i lengths; lengths
 *       [512, 300, 128] give [0, 512, 812, 940]
 *   out [total_q, num_heads, head_dim]  bf16
 *   lse [total_q, num_heads]            f32, natural-log logsumexp
 * "GQA key/value head mapping": kv_head = q_head / (num_heads / num_kv_heads),
 * num_heads % num_kv_heads == 0; K/V are never repeated in memory.
 * Scores are scaled by 1/sqrt(head_dim).  `causal` masks key j of query i
 * when j > i + (L_k - L_q) (bottom-right alignment; for L_q == L_k this is
 * j > i).  `window` > 0 keeps only the `window` most recent keys up to and
 * including the diagonal (boostr flash.rs, FlashAttentionOps docs, "Sliding
 * window"); 0 disables it.  A query with no visible key gets out = 0 and
 * lse = -inf.  lse is ln sum_j exp(q.k_j / sqrt(head_dim)) over the visible
 * keys (the quantity the backward pass of the same trait consumes).
 *
 * Memory and ownership: every pointer of varlen_attention_fwd is device
 * memory owned by the caller; nothing is retained after the call returns.
 * q, k, v, out must be 16-byte aligned, contiguous, row-major as above.  The
 * library allocates its workspace stream-ordered (cudaMallocAsync /
 * cudaFreeAsync on `stream`) and frees it on the same stream.
 *
 * Asynchrony: the call only enqueues work on `stream` (a cudaStream_t,
 * NULL = the legacy default stream) and never synchronises; cu_seqlens stay
 * on the device.  Launch errors are returned; device-side conditions (a
 * bounded barrier wait that gave up, more query tiles than max_seqlen_q
 * allows for) set bits in a device status word, which
 * varlen_attention_sync_status() reads in the order of one stream (and
 * varlen_attention_device_status() after a device-wide synchronisation).
 *
 * Preconditions not checked on the device: cu arrays are non-decreasing with
 * cu[0] = 0; max_seqlen_q / max_seqlen_k are >= every L_q / L_k (they size
 * the workspace and the tensor maps and are never used for indexing).
 * Violations can give wrong results; out-of-range rows are not read (tiles
 * past the end of the tensors are fetched with bounds-checked loads).
 *
 * Errors: each entry point returns VA_OK or a negative code and records a
 * message retrievable with varlen_attention_last_error() (per host thread).
 */
#ifndef VARLEN_ATTN_H
#define VARLEN_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VA_OK 0
#define VA_ERR_INVALID_ARG (-1) /* null pointer, negative size, H % H_kv != 0, misalignment */
#define VA_ERR_UNSUPPORTED (-2) /* head_dim other than 64 or 128, sizes beyond int32 indexing */
#define VA_ERR_CUDA (-3)        /* a CUDA runtime / driver call or a launch failed */
#define VA_ERR_DEVICE_TIMEOUT (-4) /* a bounded wait inside a kernel gave up (status queries) */

/* Device status bits (varlen_attention_device_status). */
#define VA_STATUS_WAIT_TIMEOUT 1u       /* a bounded wait inside a kernel gave up */
#define VA_STATUS_SCHEDULE_OVERFLOW 2u  /* more query tiles than max_seqlen_q allows for */
#define VA_STATUS_SMEM_ALIGN 4u         /* a backward kernel found its shared memory misaligned and did nothing */

/* Path selection for varlen_attention_fwd_ex. */
#define VA_PATH_AUTO 0    /* decode when max_seqlen_q == 1, else prefill */
#define VA_PATH_PREFILL 1 /* tensor-core tile kernel (any L_q) */
#define VA_PATH_DECODE 2  /* split-K K/V streaming kernel (requires every L_q <= 1) */

/*
 * Packed variable-length attention forward (see the file comment).
 * Argument order follows VarLenAttentionOps::varlen_attention_fwd of boostr
 * 0.2.0 varlen_attention.rs, with `window` (FlashAttentionOps "Sliding
 * window") added and the outputs passed in instead of returned.
 * head_dim must be 64 or 128.  batch == 0 or max_seqlen_q == 0 is a no-op.
 */
int varlen_attention_fwd(const void* q, const void* k, const void* v,
                         const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                         int batch, int num_heads, int num_kv_heads,
                         int max_seqlen_q, int max_seqlen_k, int head_dim,
                         int causal, int window, void* out, float* lse, void* stream);

/*
 * varlen_attention_fwd over a key-value cache with a capacity stride: the
 * packed form of the kv_seq_len argument of boostr flash.rs FlashAttentionOps
 * (section "kv_seq_len": iterate over the first n key positions while the
 * buffer's size stays the memory stride, so a full-capacity cache is passed
 * without copying).  Sequence b's slot is key/value rows cu_seqlens_k[b] ..
 * cu_seqlens_k[b+1]-1; its keys are the first min(seqused_k[b], slot size)
 * of them, and that count is the key length of the causal (bottom-right),
 * window and empty-row rules.  seqused_k is device int32 [batch], required
 * (VA_ERR_INVALID_ARG when NULL).  Slot rows past a sequence's count are
 * never visible but may be read and multiplied by exact zeros, so they must
 * hold finite values (zeros or stale keys, not NaN/inf).  max_seqlen_k bounds
 * the slot sizes.  Everything else as for varlen_attention_fwd (decode path
 * when max_seqlen_q == 1).
 */
int varlen_attention_fwd_kvcache(const void* q, const void* k, const void* v,
                                 const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                 const int32_t* seqused_k, int batch, int num_heads,
                                 int num_kv_heads, int max_seqlen_q, int max_seqlen_k,
                                 int head_dim, int causal, int window, void* out, float* lse,
                                 void* stream);

/*
 * FP8 variant: the forward pass of FlashAttentionOps::flash_attention_fwd_fp8
 * (boostr flash.rs: per-tensor dequantization scales q_scale, k_scale,
 * v_scale take the FP8 inputs to FP32, o_scale is the scale of the FP8
 * output, FP32 accumulation inside) on the packed layout of
 * varlen_attention_fwd.
 * q, k, v and out hold 8-bit E4M3 values (OCP "E4M3FN": bias 7, no
 * infinities, largest finite 448), one byte per element in the layouts of
 * the file comment; every tensor's value is code * its scale, the output's
 * included: out = E4M3(O / o_scale) with round-to-nearest-even and
 * saturation at +-448, O the attention output of the dequantized inputs (the
 * forward trait quantizes the output with o_scale, and the FP8 backward of
 * the same trait dequantizes that output with the same o_scale).  Scores are
 * (q_scale q).(k_scale k) / sqrt(head_dim); lse (f32) is the natural-log
 * logsumexp of those scores.
 * P is rounded to E4M3 before the tensor-core P V product (its row sum is
 * taken unrounded).  head_dim must be 128 (VA_ERR_UNSUPPORTED otherwise);
 * the four scales must be finite and > 0 (VA_ERR_INVALID_ARG).  Every query
 * length runs on the tensor-core tile kernel.  Memory, asynchrony and errors
 * as for varlen_attention_fwd.
 */
int varlen_attention_fwd_fp8(const void* q, const void* k, const void* v,
                             const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                             int batch, int num_heads, int num_kv_heads,
                             int max_seqlen_q, int max_seqlen_k, int head_dim,
                             int causal, int window, float q_scale, float k_scale,
                             float v_scale, float o_scale, void* out, float* lse,
                             void* stream);

/*
 * Backward pass: VarLenAttentionOps::varlen_attention_bwd of boostr 0.2.0
 * varlen_attention.rs (argument order kept: dout, q, k, v, the forward's
 * output and logsumexp, cu_seqlens, sizes, causal), with `window` as in the
 * forward (FlashAttentionOps::flash_attention_bwd of flash.rs takes it) and
 * the gradients passed in instead of returned.  Computes the gradients of
 * sum(dout * out) for the forward of varlen_attention_fwd with the same
 * masks:
 *   dq [total_q, num_heads, head_dim], dk and dv [total_k, num_kv_heads,
 *   head_dim] (GQA: summed over the query heads of each KV head), bf16.
 * dout, q, k, v, out are bf16 in the forward's layouts, lse f32
 * [total_q, num_heads] (natural log, -inf for rows with no visible key), all
 * caller-owned device memory; out and lse must be the forward's results for
 * these inputs (Delta_i = sum_d dout * out is formed from them).  Every row of
 * dq, dk, dv inside the sequences is written (zero where no visible pair
 * touches it).  head_dim 64 or 128; batch and num_heads <= 65535.  A delta
 * buffer of batch * max_seqlen_q * num_heads floats is allocated and freed
 * stream-ordered.  Asynchrony and errors as for varlen_attention_fwd.
 */
int varlen_attention_bwd(const void* dout, const void* q, const void* k, const void* v,
                         const void* out, const float* lse, const int32_t* cu_seqlens_q,
                         const int32_t* cu_seqlens_k, int batch, int num_heads, int num_kv_heads,
                         int max_seqlen_q, int max_seqlen_k, int head_dim, int causal, int window,
                         void* dq, void* dk, void* dv, void* stream);

/*
 * Same as varlen_attention_fwd with the path forced (VA_PATH_*) and, for the
 * decode path, the number of keys per split (decode_split_keys in [32, 65536];
 * 0 = library default: the largest of 4096, 2048, ..., 256 keys that still
 * gives every SM at least eight work units, counted with max_seqlen_k).  Used
 * by tests that check path and split invariance.
 */
int varlen_attention_fwd_ex(const void* q, const void* k, const void* v,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            int batch, int num_heads, int num_kv_heads,
                            int max_seqlen_q, int max_seqlen_k, int head_dim,
                            int causal, int window, void* out, float* lse,
                            int path, int decode_split_keys, void* stream);

/*
 * End-to-end variant on HOST buffers: the same operation with q, k, v,
 * cu_seqlens_q, cu_seqlens_k, out and lse all in host memory (pinned memory
 * gives asynchronous copies; pageable memory works but is staged by CUDA).
 * Copies inputs to the device, runs varlen_attention_fwd on `stream`, copies
 * out and lse back and synchronises `stream` before returning.  Device
 * buffers are allocated and freed stream-ordered inside the call.  Once the
 * inputs reach 8 MiB the batch is cut, in packed query order, into chunks of
 * about 1/16 of the query rows (at least 4096): groups of whole sequences,
 * and pieces of a longer sequence (whole 256-row query blocks with the keys
 * they can see, so a causal or windowed piece needs only the keys up to its
 * last row), pipelined: each chunk's kernels run on `stream` while the next
 * chunk's query rows and new key rows are copied in and the previous chunk's
 * results copied out on two library-owned copy streams (created on the first
 * such call per device); the results are bit-identical to one launch over the
 * whole batch.  Because both cu_seqlens arrays are in host memory here, the
 * call checks them before any device work (the checks of
 * varlen_attention_validate_cu_seqlens: cu[0] == 0, never decreasing, no
 * sequence longer than max_seqlen_q / max_seqlen_k, cu_seqlens_q[batch]
 * and cu_seqlens_k[batch] are the packed totals the copies read) and
 * returns VA_ERR_INVALID_ARG naming the first bad entry.
 */
int varlen_attention_fwd_host(const void* q, const void* k, const void* v,
                              const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                              int batch, int num_heads, int num_kv_heads,
                              int max_seqlen_q, int max_seqlen_k, int head_dim,
                              int causal, int window, void* out, float* lse, void* stream);

/*
 * Same operation as varlen_attention_fwd (always on the tensor-core prefill
 * path, which also serves single-query sequences) for callers that must not
 * allocate device memory: code inside a framework or serving runtime that
 * owns all device memory through its own allocator, or a latency-critical
 * loop that may not reach cudaMalloc or a stream-ordered allocator.  There is
 * no counterpart on the pages; it exists only for those callers.
 *
 * The call allocates nothing.  Its workspace is a static device array of
 * 1 MiB per device (every GPU that loads the library keeps it until the
 * process exits), enough for batch * ceil(max_seqlen_q / 256) <= 32760 query
 * blocks; larger problems return VA_ERR_UNSUPPORTED with a message, and
 * varlen_attention_fwd serves them.  The first call on a device performs a
 * one-time set-up with that device current (kernel attributes and the device
 * address of the static array); make that first call before any stream
 * capture.  All calls on a device share the one array and every call rewrites
 * what it reads, but calls whose work overlaps on the GPU (concurrent streams)
 * race on it: order them on one stream or serialise them.
 */
int varlen_attention_fwd_noalloc(const void* q, const void* k, const void* v,
                                 const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                 int batch, int num_heads, int num_kv_heads,
                                 int max_seqlen_q, int max_seqlen_k, int head_dim,
                                 int causal, int window, void* out, float* lse, void* stream);

/*
 * The longest-first work list the prefill path builds from cu_seqlens
 * (device pointers), written to `tiles` (device int32 [capacity][4] =
 * {sequence, query block, first key tile, end key tile}) and its length to
 * `n_tiles` (device int32).  A query block holds 256 query rows, a key tile
 * 128 keys; key tiles [first, end) hold every key any row of the block can
 * see, end == first when none.  Order: descending end - first, ties by
 * ascending (sequence, query block).  capacity must be >= the number of
 * query blocks, otherwise *n_tiles = 0 and VA_STATUS_SCHEDULE_OVERFLOW is
 * raised.
 */
int varlen_attention_schedule(const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                              int batch, int max_seqlen_q, int causal, int window,
                              int32_t* tiles, int32_t* n_tiles, int capacity, void* stream);

/*
 * Test-only export: the pipeline plan varlen_attention_fwd_host follows for
 * these host cu_seqlens arrays (host computation only, no device work).
 * input_bytes is the size of q, k and v together (the plan is one chunk below
 * 8 MiB).  Chunk c occupies chunks[9 c .. 9 c + 8] (int64): piece (1 = whole
 * 256-row query blocks of one sequence, 0 = whole sequences), b0, b1 (the
 * sequences [b0, b1)), q0, q1 (packed query rows), k_base (packed key row of
 * the chunk's key 0), k_len (a piece's key count, 0 for whole sequences),
 * kc0, kc1 (the packed key rows this chunk copies in).  Stores the number of
 * chunks in *n_chunks and writes them if capacity is at least that number.
 * Returns VA_ERR_INVALID_ARG for a NULL pointer, batch < 0, window < 0,
 * cu_seqlens that do not start at 0 or decrease, or a capacity below the
 * number of chunks (*n_chunks is still set).
 */
int varlen_attention_host_chunks(const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                 int batch, int causal, int window, long long input_bytes,
                                 long long* chunks, int capacity, int* n_chunks);

/*
 * Synchronise the current device, then store the device status word
 * (VA_STATUS_* bits, 0 = clean) in *status and, if clear != 0, reset it.
 */
int varlen_attention_device_status(unsigned* status, int clear);

/*
 * Stream-scoped status query: the device status word as seen after the work
 * already enqueued on `stream` (a cudaStream_t of the current device, NULL =
 * the legacy default stream).  Enqueues a copy of the word on `stream`,
 * synchronises that stream only (other streams keep running), stores the
 * word in *status (VA_STATUS_* bits) and, if clear != 0, resets it with a
 * write enqueued on `stream` after the copy.  The word is one per device,
 * shared by all streams: a bit raised by work on another stream shows up
 * here too once that work has finished.
 * Returns VA_ERR_DEVICE_TIMEOUT when VA_STATUS_WAIT_TIMEOUT is set (a
 * kernel's bounded wait gave up: its results are incomplete),
 * VA_ERR_CUDA when VA_STATUS_SMEM_ALIGN is set (a kernel that fills nearly all
 * of a CTA's shared memory found its base not 1024-byte aligned and wrote
 * nothing), VA_ERR_INVALID_ARG when only VA_STATUS_SCHEDULE_OVERFLOW is set (a query
 * length exceeded max_seqlen_q), VA_OK when the word is 0; VA_ERR_CUDA if a
 * copy or the synchronisation fails, VA_ERR_INVALID_ARG for a NULL status.
 * It blocks the calling host thread until `stream` drains, so it must not be
 * called while `stream` is being captured into a CUDA graph.
 */
int varlen_attention_sync_status(void* stream, unsigned* status, int clear);

/*
 * Self-test of the failure path (for tests; no fault or hang is involved).
 * Launches on `stream` a one-thread kernel that waits, through the same
 * bounded barrier wait every kernel of the library uses, on a barrier phase
 * that nothing completes.  The wait gives up after its limit (2 s of device
 * time), raises VA_STATUS_WAIT_TIMEOUT in the device status word and the
 * kernel returns normally, writing 1 to *gave_up (device int32; 0 would mean
 * the wait was satisfied).  The context stays usable afterwards.
 * Returns VA_ERR_INVALID_ARG for a NULL gave_up, VA_ERR_CUDA if the launch fails.
 */
int varlen_attention_selftest_wait_timeout(int32_t* gave_up, void* stream);

/*
 * Optional check of one cu_seqlens array against the preconditions the other
 * entry points take on trust (for tests and debugging; of the other entry
 * points only varlen_attention_fwd_host, whose arrays are already in host
 * memory, applies the same check).  cu_seqlens has batch + 1 int32 entries,
 * in host memory (on_device = 0) or in device memory (on_device != 0: copied
 * to the host on `stream`, and the calling thread then blocks until `stream`
 * drains, so a device-array check must not be made while `stream` is being
 * captured into a CUDA graph).  For the cu_seqlens_k of
 * varlen_attention_fwd_kvcache pass the largest slot size (the capacity
 * stride bound) as max_seqlen, not the largest key count in use: there the
 * steps of cu_seqlens_k are slot sizes.  Checks that cu_seqlens[0] == 0,
 * that the entries never decrease, that no sequence is longer than
 * max_seqlen and, when total >= 0, that cu_seqlens[batch] == total: the
 * packed layout of boostr varlen_attention.rs, VarLenAttentionOps docs
 * ("Layout contract": cumulative sequence lengths starting at 0).  Returns
 * VA_OK, or VA_ERR_INVALID_ARG with a message naming the first offending
 * entry (NULL pointer, batch < 0 or max_seqlen < 0 included); VA_ERR_CUDA if
 * the copy fails.  Reads nothing past entry batch.
 */
int varlen_attention_validate_cu_seqlens(const int32_t* cu_seqlens, int batch, int max_seqlen,
                                         int total, int on_device, void* stream);

/* Message for the last non-VA_OK return on this host thread ("" if none). */
const char* varlen_attention_last_error(void);

/* Library ABI version (major * 100 + minor). */
int varlen_attention_version(void);

/*
 * Diagnostic: the number of kernels this library has launched in this process
 * so far (every device and host thread; a bf16 prefill call counts its schedule
 * build and its two tile-kernel launches, an E4M3 call two, a decode call two,
 * a backward call four).  The difference across a timed region is the number
 * of the library's kernels launched in it.  Never fails.
 */
unsigned long long varlen_attention_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* VARLEN_ATTN_H */
