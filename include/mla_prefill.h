/*
 * mla_prefill.h -- C ABI of the B200 (sm_100a) varlen MLA prefill library
 * (libmla_prefill.so).
 *
 * The operation is the one the "MLA Prefill" page of the Ascend Transformer
 * Boost C API defines through AtbMLAPreFillGetWorkspaceSize / AtbMLAPreFill
 * ("Definition" section and the members table): attention of packed,
 * variable-length queries over packed keys and values, where the query-key
 * product has two parts -- the "nope" channels of Q and K (embeddimV = 128
 * wide) and the rotary channels of QRope and kRope (64 wide) -- both summed
 * into one score, scaled by qkScale (the "scaling coefficient post-multiplied
 * by Q*K^T"), masked causally (MASK_TYPE_CAUSAL_MASK in the Mask row), turned
 * into weights by a row softmax, and applied to V.  For sequence b, query
 * head h, kv head kh = h / (head_num / kv_head_num), query row i < Lq_b and
 * key j < Lk_b (Lq_b = q_seqlen[b], Lk_b = kv_seqlen[b]):
 *
 *   s_ij = qk_scale * (Q[i,h,:128] . K[j,kh,:128] + QR[i,h,:64] . KR[j,kh,:64])
 *   causal: key j is visible to row i iff j <= i + (Lk_b - Lq_b)
 *           (the mask is aligned to the bottom-right corner, so a chunk of Lq
 *           new queries sees the whole cached prefix of Lk - Lq keys)
 *   out[i,h,:] = sum_j softmax_j(s_ij) * V[j,kh,:128]     (0 if no key visible)
 *
 * The page's two-phase API (AtbMLAPreFillGetWorkspaceSize, then AtbMLAPreFill
 * with a caller-allocated workspace) is mla_prefill_get_workspace_size followed
 * by mla_prefill_ws; mla_prefill folds both into one call with a workspace the
 * library owns.  calcType is fixed to prefill, cacheMode to 0, and the Mask
 * tensor is not taken (the causal mask is computed from indices).
 */
#ifndef MLA_PREFILL_H
#define MLA_PREFILL_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream; the same type as cudaStream_t / CUstream. */
struct CUstream_st;
typedef struct CUstream_st *mla_stream_t;

/* Element types (the pages' float16 / bf16 / int8 data types, int32 lengths and tables). */
typedef enum { MLA_F16 = 0, MLA_BF16 = 1, MLA_I32 = 2, MLA_I8 = 3 } mla_dtype;

/*
 * A strided view of device memory, in the spirit of the page's aclTensor.
 * data: device pointer (caller-owned).  dtype: an mla_dtype value.
 * ndim: 1..4.  shape[d], stride[d]: extents and strides in ELEMENTS for
 * d < ndim; entries past ndim are ignored.
 */
typedef struct {
    void *data;
    int32_t dtype;
    int32_t ndim;
    int64_t shape[4];
    int64_t stride[4];
} mla_tensor;

/* maskType: the page's UNDEFINED (all-zero mask: nothing hidden) and
 * MASK_TYPE_CAUSAL_MASK (bottom-right aligned causal mask). */
typedef enum { MLA_MASK_NONE = 0, MLA_MASK_CAUSAL = 1 } mla_mask_type;

typedef enum {
    MLA_OK = 0,
    MLA_ERR_NULL = 1,          /* a required pointer is NULL */
    MLA_ERR_DTYPE = 2,         /* dtype mismatch or unsupported dtype */
    MLA_ERR_SHAPE = 3,         /* shapes inconsistent with each other / the head counts */
    MLA_ERR_ALIGN = 4,         /* base pointer not 16-byte aligned, or a stride not a multiple of 8 elements */
    MLA_ERR_HEADS = 5,         /* head_num < 1, kv_head_num < 1, or head_num % kv_head_num != 0 */
    MLA_ERR_UNSUPPORTED = 6,   /* unsupported mask type, layout or argument value */
    MLA_ERR_CUDA = 7,          /* a CUDA runtime/driver call failed */
    MLA_ERR_SEQLEN = 8,        /* device-detected: a negative seqlen, or sum(seqlen) above the tensor extent */
    MLA_ERR_DEVICE_TIMEOUT = 9, /* device-detected: a pipeline wait gave up (never expected) */
    MLA_ERR_INDEX = 10,         /* device-detected: a paged-cache block index out of range (row zeroed) */
    MLA_ERR_WORKSPACE = 11      /* caller workspace smaller than required or not 256-byte aligned */
} mla_status;

/*
 * mla_prefill -- varlen MLA prefill attention, asynchronous on `stream`.
 *
 * Inputs (all device memory, read only, one dtype: MLA_BF16 or MLA_F16):
 *   q       [T_q, H, 128] or [T_q, H*128]   Q "nope" part        (page: Q row)
 *   q_rope  [T_q, H, 64]  or [T_q, H*64]    Q rotary part        (page: QRope row)
 *   k       [T_k, G, 128] or [T_k, G*128]   K "nope" part        (page: K row, packed form)
 *   k_rope  [T_k, G, 64]  or [T_k, G*64]    K rotary part, per kv head (page: kRope row)
 *   v       [T_k, G, 128] or [T_k, G*128]   values               (page: V row, packed form)
 *     or all three in the page's padded form [batch, max_seq, G*128] / [batch,
 *     max_seq, G*64] / [batch, max_seq, G*128]: sequence b's keys are rows
 *     0 .. Lk_b-1 of batch entry b (Lk_b <= max_seq); the batch rows must be
 *     dense (batch stride = max_seq * token stride).  Rows Lk_b .. max_seq-1
 *     never reach the result, whatever they hold (NaN and Inf included).
 *     A [batch, 1, G*W] tensor reads the same either way and is taken as packed.
 *   q_seqlen, kv_seqlen  [batch] MLA_I32 in DEVICE memory (page: qSeqLen / kvSeqLen rows).
 *     Sequence b owns query tokens [sum_{b'<b} Lq_b', + Lq_b) and key tokens
 *     [sum_{b'<b} Lk_b', + Lk_b) of the packed tensors.
 *   mask_type   MLA_MASK_CAUSAL or MLA_MASK_NONE.
 *   head_num    H >= 1 (page: headNum); kv_head_num G >= 1 with H % G == 0 (page: kvHeadNum).
 *               Query head h reads kv head h / (H / G).
 *   qk_scale    any finite float (page: qkScale), multiplied onto the full two-part product.
 * Output:
 *   out     [T_q, H, 128] or [T_q, H*128], same dtype as the inputs (page: attenOut row).
 *           Rows of tokens past sum(q_seqlen) are not written.  A row with no
 *           visible key (possible when Lq_b > Lk_b) is written as zeros.
 *
 * Layout rules: the last dimension is contiguous (stride 1); token and head
 * strides are positive multiples of 8 elements (so q_rope / k_rope may be views
 * into wider buffers); every base pointer is 16-byte aligned.  K, K_rope and V
 * are either all packed or all padded (else MLA_ERR_UNSUPPORTED).  `out` must
 * not overlap any input.
 *
 * Ownership and errors: the caller owns every buffer.  Argument errors are
 * detected on the host and returned before anything is launched; `out` is then
 * untouched.  The call enqueues work on `stream` and returns without waiting.
 * The library keeps one device workspace per GPU, created on the first call on
 * that GPU and grown when a call needs more (to the need rounded up to 1 MiB).
 * Growth is stream-ordered (cudaFreeAsync / cudaMallocAsync on `stream`): the
 * call never waits on the host, but a call that grows the workspace does
 * allocate device memory.  Calls that share a GPU must be ordered on one
 * stream, or otherwise serialised, because they share that workspace; callers
 * that want concurrent streams, or no allocation at all, use mla_prefill_ws.
 * Inconsistent seqlens (negative, summing past T_q / T_k, or Lk_b > max_seq in
 * the padded form) are detected on
 * the device: the kernel clamps to the tensor extents -- it never reads or
 * writes out of bounds -- and records MLA_ERR_SEQLEN in a sticky status word
 * that mla_prefill_device_status() returns.
 * Returns MLA_OK or an mla_status error code.
 */
int mla_prefill(const mla_tensor *q, const mla_tensor *q_rope, const mla_tensor *k, const mla_tensor *k_rope,
                const mla_tensor *v, const mla_tensor *q_seqlen, const mla_tensor *kv_seqlen, int mask_type,
                int head_num, int kv_head_num, float qk_scale, mla_tensor *out, mla_stream_t stream);

/*
 * mla_prefill_get_workspace_size / mla_prefill_ws -- mla_prefill with a
 * workspace the caller allocates, in the two phases of the MLA Prefill page's
 * API (AtbMLAPreFillGetWorkspaceSize returns the workspace size for the
 * operation's arguments; AtbMLAPreFill runs it in the caller's workspace).
 *
 * mla_prefill_get_workspace_size takes the arguments of mla_prefill (only
 * their shapes, strides, dtypes and scalars are read; no device memory is
 * touched) and writes to *workspace_bytes the bytes of device memory that
 * mla_prefill_ws needs for them.  The size depends on batch, T_q, T_k (or the
 * padded form's max_seq), head_num and the split-KV choice (the calling
 * thread's mla_prefill_set_split_tiles setting and, in its automatic mode, the
 * current GPU's SM count), so both calls must see the same arguments and
 * settings.  It is at least 256 bytes.  Returns MLA_OK, an argument error as
 * mla_prefill would, MLA_ERR_NULL for a NULL workspace_bytes, or MLA_ERR_CUDA.
 *
 * mla_prefill_ws computes exactly what mla_prefill computes (the same kernels,
 * bit-identical results) using `workspace` (device memory, 256-byte aligned,
 * at least the size above, caller-owned; its previous contents do not matter)
 * for all of its scratch: it allocates nothing and never synchronises.  Calls
 * with different workspaces may run concurrently on different streams of one
 * GPU; calls that share a workspace must be ordered on one stream.  The first
 * 4 bytes of the workspace hold the call's device status (an int32 mla_status:
 * MLA_OK, MLA_ERR_SEQLEN or MLA_ERR_DEVICE_TIMEOUT), reset by each call and
 * readable once the call has completed, e.g. with mla_prefill_ws_status.
 * Returns MLA_OK, an argument error as mla_prefill would (nothing launched),
 * MLA_ERR_NULL for a NULL workspace, or MLA_ERR_WORKSPACE when the workspace
 * is too small or misaligned.
 */
int mla_prefill_get_workspace_size(const mla_tensor *q, const mla_tensor *q_rope, const mla_tensor *k,
                                   const mla_tensor *k_rope, const mla_tensor *v, const mla_tensor *q_seqlen,
                                   const mla_tensor *kv_seqlen, int mask_type, int head_num, int kv_head_num,
                                   float qk_scale, const mla_tensor *out, uint64_t *workspace_bytes);
int mla_prefill_ws(const mla_tensor *q, const mla_tensor *q_rope, const mla_tensor *k, const mla_tensor *k_rope,
                   const mla_tensor *v, const mla_tensor *q_seqlen, const mla_tensor *kv_seqlen, int mask_type,
                   int head_num, int kv_head_num, float qk_scale, mla_tensor *out, void *workspace,
                   uint64_t workspace_bytes, mla_stream_t stream);

/*
 * mla_prefill_ws_status -- synchronises `stream`, then reads the status word of
 * the last mla_prefill_ws call that used `workspace` (the int32 in its first 4
 * bytes) into *status.  Allocates nothing.  Returns MLA_OK, MLA_ERR_NULL,
 * MLA_ERR_WORKSPACE (misaligned) or MLA_ERR_CUDA.
 */
int mla_prefill_ws_status(const void *workspace, mla_stream_t stream, int *status);

/*
 * mla_prefill_device_status -- synchronises `stream`, then reads and clears the
 * device status words of the current GPU (MLA_OK, MLA_ERR_SEQLEN,
 * MLA_ERR_DEVICE_TIMEOUT or MLA_ERR_INDEX): the library's word, which
 * mla_prefill, mla_prefill_paged and mla_paged_cache_load write, and the word
 * in mla_prefill_noalloc's static array.  Each keeps the first error recorded
 * since it was last read; the library's is reported when both hold one.
 * Allocates nothing (a 4-byte copy and a 4-byte memset per word).
 * Writes it to *status and returns MLA_OK, or returns MLA_ERR_NULL /
 * MLA_ERR_CUDA.
 */
int mla_prefill_device_status(mla_stream_t stream, int *status);

/*
 * mla_prefill_noalloc -- the same operation, arguments, validation, layouts
 * and results as mla_prefill, for callers that cannot allocate device memory.
 * (The MLA Prefill page has no counterpart: its two-phase API hands the
 * operator a caller-allocated workspace; this entry point needs none.)
 *
 * Who needs it: a caller that has already reserved (nearly) all of the GPU's
 * memory for its own pool, as serving engines do at start-up, so that a
 * cudaMalloc from a library would fail or eat into that pool; and a caller
 * on a latency-critical path that must never call cudaMalloc, because a first
 * allocation or a workspace growth can stall on the driver at an arbitrary
 * moment.  mla_prefill allocates its per-GPU workspace and status word on first
 * use (and grows the workspace when a larger problem arrives); this entry point
 * calls no cudaMalloc / cudaFree or other allocating routine.
 *
 * Scratch: one static 1 MiB device array per GPU that loads the library
 * (reserved for the life of the process).  The problem must fit in it: the
 * plan workspace, 16 + 16*batch + 4*(batch+1) + 4*(ceil(T_k/128)+2) +
 * 8*(ceil(T_q/256)+batch) bytes with each part rounded up to 256 bytes, must
 * not exceed 1 MiB - 256 bytes (for example batch <= 8192 with T_q, T_k <= 1M
 * tokens fits).  A larger problem is rejected on the host with
 * MLA_ERR_UNSUPPORTED before anything is launched.
 *
 * The first call on a GPU does a one-time set-up with that GPU current (it
 * looks up the array's device address, the SM count and the tensor-map
 * encoder); make that first call before any stream capture.  All calls on a
 * GPU share the one array: calls whose work overlaps on that GPU (different
 * streams, or host threads without ordering) race and may produce wrong
 * results; order them on one stream.  Nothing in the array needs clearing
 * between calls: each call rewrites every entry it later reads.
 * Inconsistent seqlens are clamped exactly as in mla_prefill (no out-of-bounds
 * access) and recorded in a status word kept in the static array;
 * mla_prefill_device_status() reads and clears it without allocating.
 * Returns MLA_OK or an mla_status error code, like mla_prefill.
 */
int mla_prefill_noalloc(const mla_tensor *q, const mla_tensor *q_rope, const mla_tensor *k,
                        const mla_tensor *k_rope, const mla_tensor *v, const mla_tensor *q_seqlen,
                        const mla_tensor *kv_seqlen, int mask_type, int head_num, int kv_head_num, float qk_scale,
                        mla_tensor *out, mla_stream_t stream);

/*
 * mla_paged_cache_load -- gathers a block-paged key / value cache into packed
 * key / value tensors, asynchronously on `stream` (the PagedCacheLoadOperation
 * page: AtbPagedCacheLoadGetWorkspaceSize / AtbPagedCacheLoad, ND cache format).
 * Its key output, viewed as K_nope / K_rope columns, feeds mla_prefill.
 *
 *   key_cache    [num_blocks, block_size, H, Dk]  (page: keyCache, ND)
 *   value_cache  [num_blocks, block_size, H, Dv]  (page: valueCache, ND)
 *                MLA_F16, MLA_BF16 or MLA_I8 (bytes are copied, never converted);
 *                each slot's H x D block contiguous; block / slot strides free
 *                (multiples of 16 bytes); H*D*element size a multiple of 16 bytes.
 *   block_tables [batch, W] MLA_I32: logical block i of batch entry b is physical
 *                block block_tables[b][i] (page: blockTables).
 *   context_lens MLA_I32 [batch] lengths, or with context_lens_cumsum != 0,
 *                [batch + 1] running sums c with len_b = c[b+1] - c[b]
 *                (page: contextLens, isSeqLensCumsumType).
 *   seq_starts   MLA_I32 [batch] token offset of each entry's first token in
 *                its block-table row, or NULL for 0 (page: seqStarts /
 *                hasSeqStarts).
 *   key, value   [T, H, Dk] / [T, H, Dv] (or [T, H*D]) outputs, dtypes of their
 *                caches (page: key / value).  Entry b's tokens go to rows
 *                len_0 + ... + len_{b-1} onwards.
 * Token t of entry b is read from slot p % block_size of block
 * block_tables[b][p / block_size], p = seq_starts[b] + t.
 *
 * All tensors are caller-owned device memory; the outputs must not overlap
 * the caches or each other.  Argument errors return before any launch.
 * Device-detected: lengths summing past T (clamped, MLA_ERR_SEQLEN) and rows
 * whose logical block is past W or whose block id is outside [0, num_blocks)
 * (written as zeros, MLA_ERR_INDEX); read them with mla_prefill_device_status.
 * Shares the per-GPU workspace with mla_prefill: order both on one stream.
 * Returns MLA_OK or an mla_status error code.
 */
int mla_paged_cache_load(const mla_tensor *key_cache, const mla_tensor *value_cache, const mla_tensor *block_tables,
                         const mla_tensor *context_lens, const mla_tensor *seq_starts, int context_lens_cumsum,
                         mla_tensor *key, mla_tensor *value, mla_stream_t stream);

/*
 * mla_prefill_paged -- mla_prefill with K, K_rope and V read in place from
 * block-paged caches through a block table: the composition of the
 * PagedCacheLoadOperation page's gather (ND format, plain lengths, no
 * seqStarts) with the MLA Prefill page's attention, without the packed copy.
 * It runs the single-CTA attention kernel; its result is bit-identical to
 * mla_paged_cache_load into packed key / value tensors followed by mla_prefill
 * on them on that kernel (mla_prefill_set_kernel(1); the CTA-pair kernel that
 * mla_prefill picks by itself for long sequences agrees within the bound, not
 * bit for bit).
 *
 *   q, q_rope, q_seqlen, kv_seqlen, mask_type, head_num, kv_head_num,
 *   qk_scale, out   exactly as in mla_prefill.
 *   key_cache    [num_blocks, block_size, G, 192]: per slot and kv head the
 *                128 K_nope channels followed by the 64 K_rope channels
 *                (page: keyCache, ND).
 *   value_cache  [num_blocks, block_size, G, 128] (page: valueCache, ND).
 *                Both of q's dtype; last dimension contiguous; block, slot
 *                and head strides positive multiples of 8 elements; base
 *                pointers 16-byte aligned; the two caches agree in
 *                num_blocks and block_size.
 *   block_size   a multiple of 8 that divides 128, or a multiple of 128
 *                (8, 16, 32, 64, 128, 256, ...); else MLA_ERR_UNSUPPORTED.
 *   block_tables [batch, W] MLA_I32 (page: blockTables): key j < Lk_b of
 *                sequence b is slot j % block_size of physical block
 *                block_tables[b][j / block_size].  Lk_b <= W * block_size
 *                (else clamped, MLA_ERR_SEQLEN).  Entries for blocks wholly
 *                past Lk_b are never read; slots past Lk_b in the last block
 *                may hold anything (NaN and Inf included).
 *
 * All tensors are caller-owned device memory; `out` must not overlap the
 * queries or the caches.  Argument errors return before any launch.
 * Device-detected: MLA_ERR_SEQLEN as in mla_prefill, and a visible key whose
 * block id lies outside [0, num_blocks) (its K and V rows read as zeros,
 * MLA_ERR_INDEX); read them with mla_prefill_device_status.  Shares the
 * per-GPU workspace with mla_prefill: order both on one stream.
 * Returns MLA_OK or an mla_status error code.
 */
int mla_prefill_paged(const mla_tensor *q, const mla_tensor *q_rope, const mla_tensor *key_cache,
                      const mla_tensor *value_cache, const mla_tensor *block_tables, const mla_tensor *q_seqlen,
                      const mla_tensor *kv_seqlen, int mask_type, int head_num, int kv_head_num, float qk_scale,
                      mla_tensor *out, mla_stream_t stream);

/*
 * mla_prolog -- the MLA Prolog step, non-quantised (the "MlaProlog" page of
 * cann-recipes-infer: 功能说明 / 计算公式 / 参数说明 sections), asynchronous on
 * `stream`.  For each token row x of token_x:
 *
 *   c^Q = RmsNorm(x wq_a) * gamma_cq                       (stored as bf16)
 *   q   = RmsNorm(c^Q wq_b) per head, weight 1;  q[h, d-R:] = ROPE(q[h, d-R:])
 *   kv  = RmsNorm(x wkv) * gamma_ckv;            kv[d-R:]   = ROPE(kv[d-R:])
 *
 * RmsNorm(v) = v / sqrt(mean(v^2) + eps) over the row (over each head's d
 * channels for q).  ROPE is the interleaved rotation of adjacent channel pairs
 * with the token's cos / sin rows: y[2i] = v[2i] cos[2i] - v[2i+1] sin[2i],
 * y[2i+1] = v[2i+1] cos[2i+1] + v[2i] sin[2i+1].
 *
 *   token_x   [t, h]          MLA_BF16 (page: token_x)
 *   wq_a      [h, r]          MLA_BF16 (page: wq_a; r = q_lora_rank)
 *   wq_b      [r, H*d]        MLA_BF16 (page: wq_b, here unquantised; H = num_heads, d = head_dim)
 *   wkv       [h, d]          MLA_BF16 (page: wkv)
 *   rope_cos, rope_sin [t, R] MLA_BF16 (page: rope_cos / rope_sin; R = rope_dim)
 *   gamma_cq  [r], gamma_ckv [d]  MLA_BF16 (page: gamma_cq / gamma_ckv)
 *   num_heads H >= 1; eps >= 0 (not printed on the page; 1e-6 is the usual value)
 * Outputs (bf16): q_out [t, H, d] or [t, H*d] (page: q_out), kv_out [t, d]
 * (page: kv_out), and cq_out [t, r] (c^Q, the non-quantised counterpart of the
 * page's qr_out) or NULL.
 * The page's supported sizes are h 4096, r 1024, H 64, d 512, R 64, t up to
 * 64k; any sizes work with r, d, R multiples of 4 and R <= d.  Matrices have a
 * contiguous last dimension, a row stride that is a multiple of 8 elements and
 * 16-byte aligned bases; vectors are contiguous.  Outputs must not overlap each
 * other or any input.
 *
 * The q projection c^Q wq_b runs in this library's tcgen05 kernel with the
 * per-head RmsNorm and RoPE as its epilogue (the head's d channels of 256
 * tokens accumulate in fp32 in tensor memory and are written once, as bf16)
 * when d is a multiple of 128 up to 512, r a multiple of 64 and R a multiple
 * of 32 -- the
 * page's sizes among them; otherwise it runs as a library GEMM (fp32 result)
 * followed by a row kernel.  x wq_a and x wkv are library GEMMs (cuBLAS, fp32
 * results) followed by the row kernel.  Nothing is rounded before the norms
 * except c^Q, which is rounded to bf16 once before the q projection.  Scratch
 * (fp32 projections of up to 4096 tokens at a time) lives in the per-GPU
 * workspace shared with mla_prefill: order calls on one stream.  Argument
 * errors return before any launch.  Returns MLA_OK or an mla_status error code.
 */
int mla_prolog(const mla_tensor *token_x, const mla_tensor *wq_a, const mla_tensor *wq_b, const mla_tensor *wkv,
               const mla_tensor *rope_cos, const mla_tensor *rope_sin, const mla_tensor *gamma_cq,
               const mla_tensor *gamma_ckv, int num_heads, float eps, mla_tensor *q_out, mla_tensor *kv_out,
               mla_tensor *cq_out, mla_stream_t stream);

/* How this host thread's mla_prolog calls run the q projection: -1 (default)
 * the fused tcgen05 kernel wherever the sizes allow it, 0 always the library
 * GEMM followed by the row kernel (for comparison).  Returns MLA_OK, or
 * MLA_ERR_UNSUPPORTED for any other value. */
int mla_prolog_set_path(int path);

/* 1 if the last mla_prolog call of this host thread ran the fused q kernel,
 * else 0. */
int mla_prolog_last_fused(void);

/* A static, human-readable name for a status code (never NULL). */
const char *mla_status_string(int status);

/*
 * mla_prefill_set_profile_events -- profiling hook.  When both events are
 * non-NULL, every later mla_prefill call on this host thread records `start`
 * on its stream immediately before the attention kernel launch and `stop`
 * immediately after it, so the caller can time that kernel alone with
 * cudaEventElapsedTime (while the hook is on, the kernel is launched without
 * programmatic dependent launch, so none of it starts before `start`).  The
 * mla_prolog call records them around its query-row RmsNorm / RoPE launch.
 * The events are CUDA events (cudaEvent_t) owned by the caller.  Passing
 * NULL, NULL turns the hook off.  Returns MLA_OK.
 */
struct CUevent_st;
int mla_prefill_set_profile_events(struct CUevent_st *start, struct CUevent_st *stop);

/*
 * mla_prefill_set_kernel -- attention-kernel choice for later mla_prefill,
 * mla_prefill_ws and mla_prefill_noalloc calls on this host thread (no
 * counterpart on the pages; the result is the same operation either way, each
 * within the stated bound of the exact result, the two kernels' bits differing
 * where their key tiles do).
 *   kernel = -1  automatic (the default): the CTA-pair kernel for packed,
 *                unsplit K/V with long sequences (on average 3072 keys or
 *                more per sequence) once its work units (512 rows of one head,
 *                or 256 rows of two query heads sharing a kv head when each
 *                kv head serves an even number of query heads) give at least
 *                one work item per SM pair, else the single-CTA kernel;
 *   kernel =  1  the single-CTA kernel (256-row units, one SM each);
 *   kernel =  2  the CTA-pair kernel wherever it applies (packed K/V without
 *                split-KV); padded or paged K/V and split-KV always run the
 *                single-CTA kernel.
 * The CTA-pair kernel runs each unit on a cluster of two SMs: M = 256
 * tensor-core MMAs across the pair (tcgen05 cta_group::2), each SM loading half
 * of every 64-key tile, with two score buffers per 256-row group so that the
 * next tile's scores are computed during the current tile's softmax; the
 * single-CTA kernel uses 128-key tiles.  Returns MLA_OK, or MLA_ERR_UNSUPPORTED
 * for other values.
 */
int mla_prefill_set_kernel(int kernel);

/*
 * mla_prefill_set_split_tiles -- split-KV control for later mla_prefill and
 * mla_prefill_paged calls on this host thread (no counterpart on the pages).
 * A 256-row query unit normally walks all its key tiles in one work item; with
 * split-KV its key tiles go in chunks of `tiles` 128-key tiles, each chunk a
 * separate item that writes O / l and the row's log-sum-exp in fp32 to the
 * library workspace, and a combine kernel merges the chunks into attenOut
 * (the same softmax over the union of the chunks' keys).  This fills the GPU
 * when few long units exist (a long sequence at low head counts).
 *   tiles = -1  automatic (the default): split only when (units x heads) is
 *               below twice the SM count and the work is at least 16 key
 *               tiles per SM, in chunks giving ~3 items per SM;
 *   tiles =  0  never split;
 *   tiles >  0  split every unit longer than `tiles` key tiles (the chunk is
 *               doubled if the fp32 partial rows would exceed 2 GiB).
 * mla_prefill_noalloc never splits.  Returns MLA_OK, or MLA_ERR_UNSUPPORTED
 * for tiles < -1.
 */
int mla_prefill_set_split_tiles(int tiles);

/*
 * mla_selftest_wait_timeout -- diagnostic for the device timeout path (no
 * counterpart on the pages).  Launches, on `stream`, one warp that runs the
 * attention kernel's bounded pipeline wait on an mbarrier nothing arrives at,
 * with a limit of wait_ms milliseconds (1..10000) instead of the kernel's 2 s.
 * The wait gives up, records MLA_ERR_DEVICE_TIMEOUT in the device status word
 * (read it with mla_prefill_device_status) and the kernel returns: no fault,
 * no trap, and the context stays usable.  Returns MLA_OK, MLA_ERR_UNSUPPORTED
 * for wait_ms out of range, or MLA_ERR_CUDA.
 */
int mla_selftest_wait_timeout(int wait_ms, mla_stream_t stream);

/* Kernels the last mla_prefill / mla_prefill_paged / mla_prefill_noalloc call of this host thread
 * enqueued: 2 (plan + attention), 3 with split-KV (+ combine), 0 if it launched nothing. */
int mla_prefill_last_launches(void);

/* Attention kernel the last mla_prefill / mla_prefill_ws / mla_prefill_paged / mla_prefill_noalloc
 * call of this host thread launched: 1 the single-CTA kernel, 2 the CTA-pair kernel, 0 none. */
int mla_prefill_last_kernel(void);

/* Library version as 10000*major + 100*minor + patch. */
int mla_prefill_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_PREFILL_H */
