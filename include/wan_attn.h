/*
 * wan_attn.h -- C ABI of the Wan2.2 DiT self-attention hot path on B200 (sm_100a).
 *
 * The path (one DiT block's self-attention over video tokens, after the fused
 * QKV projection):
 *
 *   packed [Q|K|V] --(1) Q/K RMSNorm over the full hidden width, bf16 round,
 *                        3D RoPE, in place--> --(2) softmax attention--> out
 *
 * Sources for what is computed:
 *  - Packed storage, strided Q/K reads, in-place update that keeps the shared
 *    [Q | K | V] allocation, and the bf16 rounding point between the norm and
 *    RoPE: TensorRT-LLM PR "[visual_gen] Optimize Wan2.2 Dataflow", section 1
 *    "Preserve Packed QKV Storage Through Q/K Normalization and RoPE" and
 *    "Fused Q/K Norm and RoPE" (FP32 accumulation -> BF16 -> FP32 RoPE -> BF16).
 *  - Norm over num_heads*head_dim (5120 for A14B), weight index
 *    head*head_dim + dim: the review comments on that PR.
 *  - Token sequence S = F*H*W of the DiT grid and the bidirectional,
 *    all-pairs attention whose cost grows as S^2: AWS Neuron "Optimizing
 *    High-Quality Offline Video Generation", "Grounding in an output spec" and
 *    "Context parallelism".
 *  - 40 heads x 128 at S = 75600: the PR's "Packed QKV Profiling Details".
 *  - head_dim 128 as a requirement of the Blackwell attention path: vLLM-Omni
 *    "Wan2.2 Text-to-Video" recipe, Skip-Softmax requirements.
 *  - Error instead of silent fallback: the same recipe ("raises rather than
 *    silently degrading").
 *
 * Layouts (all row-major, bf16 = IEEE bfloat16 bit patterns):
 *  - qkv:   [batch][S][3][heads][128]. Q of (b, s, h) starts at element
 *           ((b*S + s)*3*D + h*128), K at +D, V at +2D, with D = heads*128.
 *  - out:   [batch][S][heads][128], i.e. [batch][S][D].
 *  - gamma: [D] (Q and K each), channel c = head*128 + dim.
 *  - Token s of an F x H x W grid sits at frame s/(H*W), row (s/W)%H,
 *    column s%W (width fastest).
 *
 * RoPE reading: head dims [0,44) rotate with the frame index, [44,86) with the
 * row, [86,128) with the column; pairs are adjacent elements (2i, 2i+1); the
 * j-th pair of an axis of width d_a has angle pos * theta^(-2j/d_a).
 *
 * Ownership and execution: the caller owns every buffer; the library
 * allocates no device memory (wan_dit_attn_host keeps two copy streams and
 * a pool of events per device). Calls are asynchronous on `stream` (a
 * cudaStream_t; NULL is the legacy default stream) and do not synchronise.
 * Arguments are validated before anything is launched; on any error status
 * nothing has been launched and no buffer has been written.
 *
 * Device requirement: compute capability 10.0 (B200, sm_100a); anything else
 * returns WAN_ERR_UNSUPPORTED_DEVICE. There is no fallback path.
 */
#ifndef WAN_ATTN_H_
#define WAN_ATTN_H_

#include <stdint.h>

#if defined(__GNUC__)
#define WAN_API __attribute__((visibility("default")))
#else
#define WAN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  WAN_OK = 0,
  WAN_ERR_NULL = 1,               /* a required pointer is NULL */
  WAN_ERR_ALIGN = 2,              /* a pointer is not 16-byte aligned */
  WAN_ERR_SHAPE = 3,              /* batch/grid/heads out of range, or overflow */
  WAN_ERR_HEAD_DIM = 4,           /* head_dim != 128 */
  WAN_ERR_PARAM = 5,              /* eps/theta/scale not finite or out of range */
  WAN_ERR_UNSUPPORTED_DEVICE = 6, /* current device is not compute capability 10.0 */
  WAN_ERR_LAUNCH = 7,             /* the CUDA runtime rejected a launch */
  WAN_ERR_DEVICE_TIMEOUT = 8,     /* a kernel's bounded wait gave up (see wan_device_error) */
  WAN_ERR_ALIAS = 9,              /* out overlaps qkv */
  WAN_ERR_MEMORY_KIND = 10,       /* a host buffer is not page-locked, or a device buffer
                                     is not memory of the current device */
  WAN_ERR_KERNEL_IMAGE = 11,      /* a compiled attention kernel's register count differs from
                                     the one its per-warpgroup register split was written for
                                     (a toolkit other than the one the library targets) */
  WAN_ERR_TOO_LARGE = 12,         /* the step does not fit wan_dit_attn_host_static's device
                                     buffer (WAN_HOST_STATIC_MAX_ELEMENTS) */
  WAN_ERR_BOUNDS = 13             /* a device-side index check of the debug-bounds build failed
                                     (see wan_debug_bounds) */
} wan_status;

/* wan_dit_attn_host flag: the call does not wait for earlier work on
 * `stream`. Its copies into qkv_dev still wait for the kernels of earlier
 * wan_dit_attn_host calls that read the same qkv_dev, and its kernels wait for
 * those calls' copies out of the same out_dev; nothing else orders them. The
 * caller guarantees that no other earlier work still uses qkv_dev or out_dev.
 * A caller that alternates two buffer sets between consecutive calls gets one
 * call's input transfer overlapped with the previous call's kernels. */
#define WAN_HOST_OVERLAP_INPUT 1

/* Default head-chunk size of wan_dit_attn_host's pipeline. */
#define WAN_HOST_HEADS_PER_CHUNK 8
/* Largest number of (batch element, head chunk) pieces one wan_dit_attn_host
 * call is cut into. */
#define WAN_HOST_MAX_PIECES 4096

/* Largest head count accepted (hidden width 64*128 = 8192). */
#define WAN_MAX_HEADS 64
#define WAN_HEAD_DIM 128

/* Static, human-readable text for a status code. Never NULL. */
WAN_API const char* wan_status_string(int32_t status);

/* Version of this ABI (bumped on any signature change or addition). */
WAN_API int32_t wan_abi_version(void);

/*
 * (1) Q/K RMSNorm + bf16 round + 3D RoPE, IN PLACE on the packed buffer.
 *   For every token and X in {Q, K}:
 *     r = 1/sqrt(mean_{c<D} X_c^2 + eps)      (exact squares summed in fp64)
 *     y_c = bf16_rne(X_c * r * gamma_X[c])     (correctly rounded)
 *     pairs of y rotated by the token's (frame,row,column) angles, then
 *     rounded to bf16 and written back over X: every element within 1 bf16
 *     ulp of the exact definition.
 *   V is neither read nor written.
 *   Domain: finite inputs with |X_c| < 2^64 and |X_c * gamma_X[c]| < 2^128.
 *   The squares and the gamma products are formed exactly in fp32; larger
 *   magnitudes overflow there and give wrong rows, with no error reported.
 * qkv      device pointer, bf16 [batch][F*H*W][3*heads*128], 16-byte aligned.
 * gamma_q, gamma_k  device pointers, bf16 [heads*128], 16-byte aligned.
 * batch >= 1; F, H, W >= 1 with F*H*W < 2^31; 1 <= heads <= WAN_MAX_HEADS;
 * head_dim == 128; eps > 0 finite; theta > 1 finite.
 */
WAN_API int32_t wan_qk_norm_rope(void* qkv, int64_t batch, int32_t F, int32_t H, int32_t W,
                         int32_t heads, int32_t head_dim, const void* gamma_q,
                         const void* gamma_k, float eps, float theta, void* stream);

/*
 * (2) Full bidirectional softmax attention per (batch, head), reading Q, K and
 *   V straight from the packed buffer (no repack):
 *     out[b, i, h, :] = sum_j softmax_j(scale * q_i . k_j) v_j
 *   bf16 operands, fp32 accumulation, probabilities rounded to bf16 before
 *   the PV product, output rounded to bf16.
 *   Domain: finite inputs whose scores scale * q_i . k_j and weighted sums stay
 *   finite in fp32, where the tensor cores accumulate them (inputs normalised
 *   by (1) are bounded by sqrt(heads*128) * max|gamma| per element).
 * qkv      device pointer, bf16 [batch][seq_len][3*heads*128], 16-byte aligned.
 * out      device pointer, bf16 [batch][seq_len][heads*128], 16-byte aligned,
 *          must not overlap qkv.
 * scale    > 0, or <= 0 to mean 1/sqrt(head_dim).
 * batch >= 1, 1 <= seq_len < 2^31, 1 <= heads <= WAN_MAX_HEADS, head_dim == 128.
 */
WAN_API int32_t wan_self_attention(const void* qkv, void* out, int64_t batch, int64_t seq_len,
                           int32_t heads, int32_t head_dim, float scale, void* stream);

/*
 * (2) with Skip-Softmax in threshold mode (vLLM-Omni "Wan2.2 Text-to-Video"
 * recipe, "Accelerating with TRTLLM_ATTN + Skip-Softmax": a direct skip
 * threshold, no calibration; the output diverges from dense as the
 * threshold grows). Rule, per query tile of 128 rows and key tile j >= 1 of
 * 128 keys, in groups of 32 query rows: a group skips key tile j when each of
 * its rows has every weight of the tile below threshold x the row's largest
 * weight over key tiles 0..j-1 (in scores: tile max < running max +
 * ln(threshold)). A skipped tile adds nothing to the group's row sums and
 * weighted sums; when all four groups of a query tile skip, the P V product
 * is not run. Tile 0 is never skipped; a group holding rows past seq_len
 * never skips. threshold == 0 runs the dense kernel (bit-identical to
 * wan_self_attention); 0 <= threshold <= 1 (a weight is compared with the
 * row's largest one, so a threshold above 1 would also drop tiles that hold
 * the row's maximum), else WAN_ERR_PARAM.
 * Other arguments as for wan_self_attention. Counters of what was skipped:
 * wan_skip_stats.
 */
WAN_API int32_t wan_self_attention_sparse(const void* qkv, void* out, int64_t batch, int64_t seq_len,
                                          int32_t heads, int32_t head_dim, float scale, float threshold,
                                          void* stream);

/*
 * FP8 (e4m3) variant of (2) -- the attention arithmetic the pages time (Neuron
 * "Optimizing High-Quality Offline Video Generation"; the TensorRT-LLM PR's TE
 * FP8 attention profile) -- with per-tensor scales. A tensor X is stored as
 * codes c = e4m3(fl32(x * inv_scale_X)) (round to nearest even, saturating at
 * +-448) and stands for c * scale_X; the caller picks the scales (typically
 * scale_X = amax_X / 448 from wan_qkv_amax, inv_scale_X = 1 / scale_X).
 *
 * wan_qkv_amax: max |x| of Q, K and V of the packed bf16 buffer into
 *   amax[0..2] (device pointer to 3 floats, 4-byte aligned), asynchronously.
 * wan_quantize_fp8: codes of the packed bf16 buffer:
 *   qk8  device, [batch][seq_len][2][heads][128] e4m3 (Q then K per token);
 *   v8t  device, [batch][heads][128][s_pitch] e4m3: V transposed per
 *        (batch, head), key-contiguous; columns past seq_len hold code 0;
 *   s_pitch: a multiple of 16, >= seq_len. Both 16-byte aligned.
 * wan_self_attention_fp8: out[b, i, h, :] = sum_j softmax_j(scale * q_i . k_j) v_j
 *   on the dequantised operands, both products in kind::f8f6f4 on the tensor
 *   cores (fp32 accumulation), the probabilities rounded to e4m3 for the P V
 *   product, out in bf16 [batch][seq_len][heads*128]. scale <= 0 means
 *   1/sqrt(128). The e4m3 rounding of the operands and of P makes the result
 *   differ from the bf16 path by a few per cent (relative Frobenius).
 * Scales finite and > 0; head_dim == 128; buffers must not overlap out.
 */
WAN_API int32_t wan_qkv_amax(const void* qkv, int64_t batch, int64_t seq_len, int32_t heads, int32_t head_dim,
                             float* amax, void* stream);
WAN_API int32_t wan_quantize_fp8(const void* qkv, void* qk8, void* v8t, int64_t batch, int64_t seq_len,
                                 int32_t heads, int32_t head_dim, int64_t s_pitch, float inv_scale_q,
                                 float inv_scale_k, float inv_scale_v, void* stream);
WAN_API int32_t wan_self_attention_fp8(const void* qk8, const void* v8t, void* out, int64_t batch,
                                       int64_t seq_len, int32_t heads, int32_t head_dim, int64_t s_pitch,
                                       float scale, float scale_q, float scale_k, float scale_v, void* stream);

/*
 * The DiT block's projections (the third NEXT item): Y = X W^T on the tensor
 * cores (tcgen05, bf16 operands, fp32 accumulation, bf16 output), X [M][K],
 * W [N][K] (a Linear layer's weight), Y [M][N], all device, 16-byte aligned,
 * N a multiple of 256, K a multiple of 64, Y overlapping neither input. For
 * the QKV projection (N = 3*heads*128, Y the packed buffer) the epilogue can
 * fuse the Q/K RMSNorm's statistic (the Neuron page's qkv_cte fuses the
 * projection with the distributed QK RMSNorm, "NKI kernels"): when stats is
 * not NULL, stats[row][j] = the fp64 sum of squares of the bf16 outputs of
 * row `row` in columns [256 j, 256 j + 256) (a zero output counting 2^-127,
 * as in (1)'s own sum; exact for outputs below 2^64 in magnitude, the domain
 * of (1)), for j < stat_cols / 256
 * (stat_cols a multiple of 256, <= N; stats 8-byte aligned, [M][stat_cols/256]).
 */
WAN_API int32_t wan_linear(const void* x, const void* w, void* y, int64_t M, int64_t N, int64_t K,
                           double* stats, int64_t stat_cols, void* stream);

/*
 * (1) with the row statistics of the QKV projection: as wan_qk_norm_rope, but
 * each token's sum of squares of Q (and of K) is the sum of its stats entries
 * (wan_linear with stat_cols = 2*heads*128 on the same buffer) instead of a
 * reduction over the row. stats: device, [batch*F*H*W][2*heads*128/256] fp64.
 */
WAN_API int32_t wan_qk_norm_rope_stats(void* qkv, int64_t batch, int32_t F, int32_t H, int32_t W, int32_t heads,
                                       int32_t head_dim, const void* gamma_q, const void* gamma_k, float eps,
                                       float theta, const double* stats, void* stream);

/*
 * Sequence parallelism (the fourth NEXT item; Neuron page, "Context
 * parallelism": each rank owns S/N tokens, and its queries must attend every
 * key). Two calls make a rank's share of the path:
 * wan_qk_norm_rope_shard: (1) on a buffer holding tokens [s0, s0 + s_local)
 *   of every batch element's F x H x W grid ([batch][s_local][3*heads*128];
 *   RoPE positions from the grid index s0 + i). 0 <= s0, s0 + s_local <= F*H*W.
 * wan_self_attention_rows: (2) for query rows [q_row0, q_row0 + q_rows) of the
 *   full packed buffer qkv ([batch][seq_len][3*heads*128], every key present,
 *   e.g. after an all-gather of the normalised shards); out holds q_rows rows
 *   per batch element ([batch][q_rows][heads*128]). 0 <= q_row0,
 *   q_row0 + q_rows <= seq_len.
 * The bits equal those of the unsharded calls for the same rows.
 */
WAN_API int32_t wan_qk_norm_rope_shard(void* qkv, int64_t batch, int32_t F, int32_t H, int32_t W, int64_t s0,
                                       int64_t s_local, int32_t heads, int32_t head_dim, const void* gamma_q,
                                       const void* gamma_k, float eps, float theta, void* stream);
WAN_API int32_t wan_self_attention_rows(const void* qkv, void* out, int64_t batch, int64_t seq_len, int32_t heads,
                                        int32_t head_dim, int64_t q_row0, int64_t q_rows, float scale, void* stream);

/*
 * Context parallelism in ring form (the fourth NEXT item; AWS Neuron page,
 * "Context parallelism" and "NKI kernels": each rank keeps its S/N shard of Q
 * and of K/V, the K/V chunks travel around the ring, and each round's
 * attention, overlapped with the next exchange, is folded into the rank's
 * running result; the page's kernel for this is ring_attention_const_max_fwd).
 * A round's result is the online-softmax state of one key range, and states
 * over disjoint ranges combine exactly:
 *
 * wan_self_attention_partial: (2) for query rows [q_row0, q_row0 + q_rows) of
 *   q_qkv (packed, [batch][q_seq_len][3*heads*128]) against the keys
 *   [k_row0, k_row0 + k_rows) of kv ([batch][kv_rows][kv_pitch] bf16 whose
 *   last 2*heads*128 columns hold K then V: kv_pitch = 3*heads*128 for a packed
 *   QKV buffer, 2*heads*128 for a K|V chunk). Instead of the normalised bf16
 *   output it writes the softmax state of that key range, per (row, head):
 *     o  [batch][q_rows][heads][128] fp32: O = sum_j 2^(a_j - m) v_j
 *     ml [batch][q_rows][heads][2]   fp32: (m, l = sum_j 2^(a_j - m))
 *   with a_j = scale * log2(e) * q . k_j (scale <= 0: 1/sqrt(128)) and m a
 *   reference maximum chosen by the kernel (at most 8 below the largest a_j).
 *   O uses the probabilities rounded to bf16, as (2) does, and so does l.
 *   All pointers 16-byte aligned; o and ml overlap neither input nor each
 *   other. The full row's output is merge(all ranges) finalised below.
 * wan_self_attention_accumulate: as wan_self_attention_partial, but o and ml
 *   already hold a state (over other keys, e.g. earlier ring rounds), and the
 *   launch merges its own state into them (the merge below, done in the
 *   attention's epilogue) instead of overwriting them: one launch per ring
 *   round after the first, with no separate merge and no buffer for the
 *   round's own state.
 * wan_attention_merge: for n_units (row, head) units in the layouts above
 *   (n_units = batch * rows * heads): when o_part is not NULL,
 *   (o_acc, ml_acc) := the merge of itself and (o_part, ml_part):
 *     m = max(m_acc, m_part), O = 2^(m_acc - m) O_acc + 2^(m_part - m) O_part,
 *     l likewise;
 *   then, when out is not NULL, out = bf16(O_acc / l_acc), 128 bf16 per unit
 *   (for units ordered [batch][rows][heads]: wan_self_attention's layout).
 *   o_part and ml_part are both given or both NULL; o_part and out are not
 *   both NULL. No buffer overlaps another. head_dim == 128.
 */
WAN_API int32_t wan_self_attention_partial(const void* q_qkv, int64_t q_seq_len, int64_t q_row0, int64_t q_rows,
                                           const void* kv, int64_t kv_rows, int64_t kv_pitch, int64_t k_row0,
                                           int64_t k_rows, float* o, float* ml, int64_t batch, int32_t heads,
                                           int32_t head_dim, float scale, void* stream);
WAN_API int32_t wan_self_attention_accumulate(const void* q_qkv, int64_t q_seq_len, int64_t q_row0,
                                              int64_t q_rows, const void* kv, int64_t kv_rows, int64_t kv_pitch,
                                              int64_t k_row0, int64_t k_rows, float* o, float* ml, int64_t batch,
                                              int32_t heads, int32_t head_dim, float scale, void* stream);
WAN_API int32_t wan_attention_merge(float* o_acc, float* ml_acc, const float* o_part, const float* ml_part,
                                    void* out, int64_t n_units, int32_t head_dim, void* stream);

/*
 * Reads and clears the Skip-Softmax counters: *group_tiles = (32-row group,
 * key tile) pairs skipped, *products = 128-row P V products skipped. The
 * counters are one pair per device, shared by every wan_self_attention_sparse
 * launch on it (any stream, any host thread): a read returns what all of them
 * counted since the previous read. The read and the clear are one atomic
 * exchange, done on `stream` after the work enqueued on it before this call;
 * the call then synchronises `stream`. Either pointer may be NULL. Returns
 * WAN_ERR_LAUNCH when the stream reports a CUDA error.
 */
WAN_API int32_t wan_skip_stats(void* stream, int64_t* group_tiles, int64_t* products);

/*
 * (1) then (2) on one stream, the second launch chained to the first with
 * programmatic dependent launch so its prologue overlaps the first's tail.
 * Same arguments and in-place semantics as the two calls above, with
 * seq_len = F*H*W. All arguments are validated before either launch.
 */
WAN_API int32_t wan_dit_attn(void* qkv, void* out, int64_t batch, int32_t F, int32_t H, int32_t W,
                     int32_t heads, int32_t head_dim, const void* gamma_q, const void* gamma_k,
                     float eps, float theta, float scale, void* stream);

/*
 * (1) then (2) for packed QKV and output that live in HOST memory: the call
 * a user with host-resident activations makes. The PCIe transfers and the
 * kernels bound this step about equally, so they overlap:
 *  - each batch element's packed rows are copied in one contiguous copy (the
 *    fastest pattern over PCIe), and (1) runs on the element once they have
 *    arrived, while the next element's copy proceeds;
 *  - (2) follows in chunks of heads_per_chunk heads, and each head chunk of
 *    `out` is copied back while later chunks compute;
 *  - with WAN_HOST_OVERLAP_INPUT, consecutive calls on alternating buffer
 *    sets also overlap one call's copies with the previous call's kernels.
 * qkv_host  page-locked host memory (cudaHostAlloc / cudaHostRegister), bf16
 *           [batch][F*H*W][3*heads*128]; only read.
 * out_host  page-locked host memory, bf16 [batch][F*H*W][heads*128]; written.
 * qkv_dev   device memory of the current device, same shape as qkv_host:
 *           receives the copy and is normalised in place (left holding the
 *           normalised Q|K and V).
 * out_dev   device memory of the current device, same shape as out_host,
 *           must not overlap qkv_dev.
 * heads_per_chunk  1..heads, or 0 for WAN_HOST_HEADS_PER_CHUNK (capped at
 *           heads); batch * ceil(heads/heads_per_chunk) <= WAN_HOST_MAX_PIECES.
 * flags     0 or WAN_HOST_OVERLAP_INPUT.
 * Other arguments as for wan_dit_attn. Device pointers 16-byte aligned.
 * Execution: asynchronous. The call's copies and kernels start after the work
 * enqueued on `stream` before it (unless WAN_HOST_OVERLAP_INPUT), and work
 * enqueued on `stream` after it runs once out_host is written (synchronise
 * `stream` before reading out_host on the host). The library runs the copies
 * in and out and the kernels on three internal streams per device. Calls on
 * one device are serialised while they are enqueued, and their kernels run in
 * that order.
 * Ownership: all four buffers stay the caller's. They must stay allocated, and
 * qkv_host unmodified, until `stream` has passed this call: the copies read
 * qkv_host and write out_host after the call returns. A pinned-memory cache
 * that recycles a freed block at once (as PyTorch's does for memory it did not
 * see in use) must not get qkv_host back before then.
 * Errors: argument errors return before anything is enqueued, as for the other
 * calls; WAN_ERR_MEMORY_KIND when a host buffer is not page-locked or a device
 * buffer is not memory of the current device; WAN_ERR_LAUNCH when the runtime
 * rejects a copy or launch while enqueueing (part of the step may then be
 * enqueued already).
 */
WAN_API int32_t wan_dit_attn_host(const void* qkv_host, void* out_host, void* qkv_dev, void* out_dev,
                                  int64_t batch, int32_t F, int32_t H, int32_t W, int32_t heads,
                                  int32_t head_dim, const void* gamma_q, const void* gamma_k,
                                  float eps, float theta, float scale, int32_t heads_per_chunk,
                                  int32_t flags, void* stream);

/* Largest batch * F*H*W * heads * 128 that wan_dit_attn_host_static takes:
 * its device buffer holds 8 bytes per element (packed QKV, 6, and the
 * output, 2), 64 MiB in all. */
#define WAN_HOST_STATIC_MAX_ELEMENTS (8 * 1024 * 1024)

/*
 * wan_dit_attn_host for callers that cannot allocate device memory. This
 * entry point has no counterpart on the pages; it is the host-buffer step
 * with its device staging in memory the library owns.
 *
 * Why: some callers have no way to get device memory for the staging buffers
 * that wan_dit_attn_host asks for. One example is a host application that
 * hands this library only host buffers and owns no device allocator. Another
 * is a process whose device memory is reserved by another runtime's pool,
 * where cudaMalloc would fail. A third is a latency-bound caller that cannot
 * afford cudaMalloc's implicit device-wide synchronisation. This call
 * allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 * routine.
 *
 * The staging is a fixed array of device memory inside the library,
 * 8 * WAN_HOST_STATIC_MAX_ELEMENTS bytes (64 MiB). Every GPU that loads the
 * library holds its copy of the array until the process exits.
 * batch * F*H*W * heads * 128 above WAN_HOST_STATIC_MAX_ELEMENTS returns
 * WAN_ERR_TOO_LARGE before anything is launched.
 *
 * The first call on a device looks up the array's device address, with that
 * device current. The first call also creates the pipeline's internal
 * streams and events, as wan_dit_attn_host's first call does. Make that first
 * call on each device before any stream capture.
 *
 * Every call uses the same array, and the array keeps the last call's
 * contents: its packed QKV after norm+RoPE, and its output. Nothing in the
 * array has to start at zero, because each call overwrites what it reads.
 * Two calls that used the array at the same time on the GPU would overwrite
 * each other's data, so they must not overlap there. The library keeps them
 * apart: each call's copies and kernels wait for the previous call's use of
 * the array, through the same per-buffer ordering that wan_dit_attn_host
 * applies to a reused pair of device buffers. Calls from several host
 * threads or streams are therefore serialised on the device, and
 * WAN_HOST_OVERLAP_INPUT gains no overlap here.
 *
 * Arguments, layouts, execution and errors are those of wan_dit_attn_host
 * without qkv_dev and out_dev. qkv_host and out_host are page-locked host
 * memory (WAN_ERR_MEMORY_KIND otherwise). gamma_q and gamma_k are device
 * pointers, as before.
 */
WAN_API int32_t wan_dit_attn_host_static(const void* qkv_host, void* out_host, int64_t batch, int32_t F, int32_t H,
                                         int32_t W, int32_t heads, int32_t head_dim, const void* gamma_q,
                                         const void* gamma_k, float eps, float theta, float scale,
                                         int32_t heads_per_chunk, int32_t flags, void* stream);

/*
 * Reads and clears the device-side error words that the kernels set when one
 * of their bounded waits gives up. *code receives 0 when no wait gave up,
 * otherwise a nonzero value: the bf16 attention's site code in bits 0-7,
 * norm+RoPE's in bits 8-15, the FP8 attention's in bits 16-23, the projection
 * GEMM's in bits 24-30. The words are one set per device, shared by every
 * launch on it (any stream, any host thread): a read reports and clears what
 * any of them recorded since the previous read, so a caller that needs to
 * know which call failed keeps other work off the device meanwhile. The read
 * and the clear are one atomic exchange per word, done on `stream` after the
 * work enqueued on it before this call; the call then synchronises `stream`.
 * Returns WAN_ERR_DEVICE_TIMEOUT when *code != 0, WAN_ERR_NULL when code is
 * NULL, WAN_ERR_LAUNCH when the stream reports a CUDA error.
 */
WAN_API int32_t wan_device_error(void* stream, int32_t* code);

/*
 * Debug-bounds build (libwanattn_debug.so, compiled with WAN_DEBUG_BOUNDS):
 * every instrumented global- and shared-memory access of the kernels checks
 * its element range against the extent of its buffer as the launch
 * parameters define it; a failed check records the site and offset, counts
 * the failure and skips the access (no trap: the context stays usable). The
 * pages have no counterpart: this stands in for a memory checker, which this
 * library cannot rely on being available.
 *
 * Synchronises `stream`, then reads and clears the records of every kernel
 * file. *enabled = 1 in the debug-bounds build, 0 in the release build (which
 * records nothing and touches no device). *first_fault is 0 when no check
 * failed, else the first failure of the first kernel file that has one: the
 * site in bits 56-63 (debug_bounds.cuh names them) and the element offset's
 * low 56 bits; *count is the number of failed checks. Like wan_device_error's
 * words, the records are one set per device, shared by every launch on it.
 * Returns WAN_ERR_BOUNDS when *count != 0, WAN_ERR_NULL when a pointer is
 * NULL, WAN_ERR_LAUNCH when a CUDA call fails.
 */
WAN_API int32_t wan_debug_bounds(void* stream, int32_t* enabled, uint64_t* first_fault, uint64_t* count);

/*
 * Self-test of failure detection. Launches the attention kernel exactly as
 * wan_self_attention does, except that its producer starts no copies, so
 * every bounded wait of the kernel runs out after `wait_limit_ns`
 * (1e3 .. 2e9 ns). The kernel then records the timeout in its device error
 * word, drains, releases its tensor memory and exits without touching `out`.
 * Read the result with wan_device_error (expected: WAN_ERR_DEVICE_TIMEOUT with
 * a nonzero site code); the CUDA context stays usable. This is how a stalled
 * pipeline surfaces as an error instead of a hang (the vLLM-Omni recipe's
 * rule that the backend raises rather than silently degrading).
 * Arguments as for wan_self_attention; nothing is written to qkv or out.
 */
WAN_API int32_t wan_selftest_wait_timeout(const void* qkv, void* out, int64_t batch, int64_t seq_len,
                                          int32_t heads, int32_t head_dim, int64_t wait_limit_ns,
                                          void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WAN_ATTN_H_ */
