/*
 * pagedattn.h -- C ABI of libpagedattn: paged-attention decode on one
 * NVIDIA B200 (sm_100a).
 *
 * The operation (gllm PR #116 "feat(backend): sliding-window
 * PagedAttention", section "What changes", Interface):
 *
 *   PagedAttention(dst, q, kCache, vCache, blockTables, seqLens, queryLens,
 *                  scale, window)
 *
 * For every row b with queryLens[b] = L > 0, every query token i < L and every
 * query head h:
 *   p   = seqLens[b] - L + i          (the L new tokens are the last L of
 *                                      the row's seqLens[b] cached tokens)
 *   lo  = window > 0 ? max(0, p + 1 - window) : 0,   hi = p + 1
 *   g   = h / (H_q / H_kv)            (grouped-query heads; ExecuTorch PR
 *                                      #18759, sdpa_decode_splitk docstring)
 *   k_t = kCache[blockTables[b][t / BS]][g][t % BS][:]   (same for v_t)
 *   dst[b,i,h,:] = sum_{t in [lo,hi)} softmax_t(scale * q[b,i,h,:] . k_t) v_t
 *
 * Long spans are cut into split-K partitions whose partial results are merged
 * by a log-sum-exp reduce (ExecuTorch PR #18759, split-K flash-decoding and
 * its reduce kernel); when one partition suffices the kernel writes dst
 * directly and needs no temporaries (aiter PR #2914 "Pa gluon swa mtp opt",
 * the one_shot path).
 *
 * FP8 operands (aiter PR #2914 "Pa gluon swa mtp opt", the review of
 * pa_decode_gluon's scale arguments: an FP8 query comes with query_scale, FP8
 * KV caches with key_scale and value_scale, and a missing scale must be
 * rejected rather than silently ignored).  With pa_params.kv_dtype = PA_DTYPE_FP8_E4M3 the caches hold FP8
 * e4m3 codes (OCP 8-bit format: 1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits, no infinities) and k_t, v_t above are the codes' values
 * times the per-tensor k_scale, v_scale; with q_dtype = PA_DTYPE_FP8_E4M3, q
 * holds codes and q is their value times q_scale.  dst stays bf16.
 *
 * Layouts (all row-major, element type bf16 unless noted; FP8 codes are one
 * byte each, in the same shapes):
 *   q, dst        [sum(queryLens)][H_q][head_dim], rows packed in batch order
 *   kCache,vCache [num_blocks][H_kv][kvBlockSize][head_dim]
 *   blockTables   int32 [batch][max_blocks_per_seq]; only the first
 *                 ceil(seqLens[b] / kvBlockSize) entries of row b are read
 *   seqLens, queryLens, windows  int32 [batch]
 *
 * Ownership: the caller owns every buffer, including the workspace; the
 * library allocates no device memory in pa_decode.  All calls are
 * asynchronous on the given stream (a cudaStream_t passed as void*, NULL for
 * the legacy default stream) except where stated.
 *
 * Errors: every entry point returns PA_OK or a PA_ERR_* code and leaves a
 * one-line message for pa_last_error().  Conditions only the device can see
 * (a row with queryLen > seqLen, a block-table entry outside the pool, a
 * length beyond the caller's hints, a wait that timed out) skip the affected
 * work and set bits in a device status word read by pa_device_status().
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define PA_OK 0
#define PA_ERR_ARG 1          /* invalid argument (null pointer, bad size, misalignment) */
#define PA_ERR_UNSUPPORTED 2  /* valid but not built: head_dim or block size */
#define PA_ERR_WORKSPACE 3    /* workspace missing or smaller than pa_workspace_size */
#define PA_ERR_CUDA 4         /* a CUDA runtime call failed */

/* Device status bits (pa_device_status). */
#define PA_DEV_TIMEOUT 1u     /* a bounded wait gave up (~1 s, or the wait_limit_cycles knob) */
#define PA_DEV_BAD_ROW 2u     /* queryLens[b] > seqLens[b], negative length or window */
#define PA_DEV_BAD_BLOCK 4u   /* a block-table entry outside [0, num_blocks) */
#define PA_DEV_HINT 8u        /* a row longer than max_span_hint / max_query_len_hint */

/* Operand types (pa_params.q_dtype, pa_params.kv_dtype). */
#define PA_DTYPE_BF16 0
#define PA_DTYPE_FP8_E4M3 1   /* per-tensor scaled FP8 e4m3 codes (tensor-core variant) */

/* Scheduling of a call (pa_params.schedule). */
#define PA_SCHED_STATIC 0     /* default: one CTA per fixed partition, then the reduce kernel */
#define PA_SCHED_WORKLIST 2   /* one launch: a one-wave cooperative grid whose CTAs claim each
                                 unit's 64-token stages from a work-list counter and merge their
                                 own partials (PA_VARIANT_MMA only; see pa_params.schedule) */

/* Kernel variants (pa_params.force_variant, pa_plan_info.variant). */
#define PA_VARIANT_AUTO 0
#define PA_VARIANT_FMA 1      /* CUDA-core FMA scores and PV (group x queryLen <= 4 rows) */
#define PA_VARIANT_MMA 2      /* tensor-core m16n8k16 tiles with TMA-swizzled staging (dense rows) */
#define PA_VARIANT_TC 3       /* tcgen05 MMAs on FP8 codes in shared memory, accumulators in tensor
                                 memory (FP8 caches, head_dim 128; 8 rows per CTA) */

typedef struct pa_params {
    int batch;               /* rows */
    int num_q_heads;         /* H_q, a multiple of num_kv_heads */
    int num_kv_heads;        /* H_kv */
    int head_dim;            /* 64, 128 or 256 (256: tensor-core variant) */
    int num_blocks;          /* KV pool size in blocks */
    int max_blocks_per_seq;  /* blockTables row stride (entries) */
    /* Host hints.  max_span_hint >= max_b union span, where a row's union
     * span is seqLen - max(0, seqLen - queryLen + 1 - window) for window > 0
     * and seqLen otherwise; max_query_len_hint >= max_b queryLens[b].  With
     * both set pa_decode never synchronises.  0 means unknown: pa_decode then
     * copies the lengths to the host once (a stream synchronisation). */
    int max_span_hint;
    int max_query_len_hint;
    const int32_t *windows;  /* device [batch] per-row windows, or NULL for the scalar window */
    void *workspace;         /* device, >= pa_workspace_size() bytes when that is > 0 */
    size_t workspace_bytes;
    int force_variant;       /* PA_VARIANT_AUTO, or a PA_VARIANT_* for tests and A/B runs */
    int force_partitions;    /* 0 = dispatcher's choice; n > 0 cuts the longest span into ~n partitions */
    /* Optional instrumentation: NULL, or a host array of two cudaEvent_t that
     * pa_decode records on the stream immediately before and after the
     * partition kernel (the reduce, if any, runs after the second). */
    void *const *profile_events;
    /* Operand types: PA_DTYPE_BF16 (0, the default) or PA_DTYPE_FP8_E4M3.
     * A scale is read only for an FP8 operand and must then be finite and
     * > 0: the zero of a zero-initialised struct means "not given" and is
     * rejected.  FP8 runs on the tensor-core variant only (force_variant FMA
     * with an FP8 operand is PA_ERR_UNSUPPORTED); with FP8 caches its MMAs
     * take f16 operands, so a bf16 q must lie within f16's range (|q| <
     * 65504). */
    int q_dtype;
    int kv_dtype;
    float q_scale;
    float k_scale;
    float v_scale;
    /* PA_SCHED_*; 0 = PA_SCHED_STATIC.  PA_SCHED_WORKLIST (aiter PR #2914's
     * persistent-scheduling idea, on one wave): one launch whose CTAs take a
     * unit's stages in arrival order from a counter in the workspace and
     * merge the unit's partials themselves after an arrival count, so no
     * reduce kernel runs.  It needs PA_VARIANT_MMA and a grid that
     * fits the GPU at once (PA_ERR_UNSUPPORTED otherwise, PA_ERR_CUDA if the
     * cooperative launch is refused).  The counters are tagged with a
     * per-call epoch and need no initialisation; calls that share a
     * workspace must not overlap, and a call on a stream that is being
     * captured into a CUDA graph fails with PA_ERR_UNSUPPORTED (a replay
     * would repeat the epoch).  Results can differ from the static
     * schedule's in the last bits (the stages' grouping depends on timing),
     * and it measures slower on the named workloads, so it is opt-in. */
    int schedule;
    /* Test knobs of the one wait on other CTAs, the work-list merge's wait
     * for its unit's arrivals (0 = off, the default).  wait_limit_cycles > 0
     * replaces that wait's ~1 s limit (SM clock cycles); merge_target_extra
     * > 0 raises the arrival count it waits for, so the count is never met:
     * the wait gives up at the limit, the kernel returns, PA_DEV_TIMEOUT is
     * set and the unit's dst rows are left unwritten.  The waits for the
     * kernels' own bulk copies keep their fixed limit. */
    long long wait_limit_cycles;
    int merge_target_extra;
} pa_params;

/* What the dispatcher chose for a call (pa_plan). */
typedef struct pa_plan_info {
    int variant;             /* PA_VARIANT_* */
    int partition_tokens;    /* tokens per split-K partition (multiple of 64) */
    int max_partitions;      /* partitions of the longest span (1 = one-shot) */
    int one_shot;            /* 1: every row fits one partition, no workspace, no reduce */
    int max_rows;            /* rows per (row, kv head) unit: (H_q/H_kv) * max queryLen */
    int slab_rows;           /* rows one CTA handles; units with more rows use several CTAs */
    int consumer_warps;      /* compute warps per CTA (plus one copy warp) */
    int stages;              /* shared-memory pipeline depth */
    int grid_x, grid_y, grid_z;
    int block_threads;
    size_t smem_bytes;
    size_t workspace_bytes;  /* 0 when one_shot */
    int num_sms, ctas_per_sm;
    int worklist;            /* 1: work-list schedule (no reduce launch) */
} pa_plan_info;

/*
 * pa_decode -- paged-attention decode (the operation at the top of this file).
 *
 *   dst          device bf16 [sum(queryLens)][H_q][head_dim], written for rows
 *                with queryLens[b] > 0; other memory is untouched
 *   q            device bf16 (or FP8 codes, q_dtype) [sum(queryLens)][H_q][head_dim]
 *   kCache,vCache device bf16 (or FP8 codes, kv_dtype) [num_blocks][H_kv][kvBlockSize][head_dim]
 *   blockTables  device int32 [batch][max_blocks_per_seq]
 *   seqLens      device int32 [batch], cached tokens per row (includes the new ones)
 *   queryLens    device int32 [batch], new query tokens per row (0 skips the row)
 *   scale        multiplies q.k, used exactly as given
 *   window       0 = full causal; w > 0 = each token sees its last w positions;
 *                overridden per row by params->windows when that is not NULL
 *   kvBlockSize  tokens per KV block: a power of two in [16, 1024]
 *   params       dimensions, hints, workspace (see pa_params)
 *   stream       cudaStream_t
 *
 * All device pointers must be 16-byte aligned.  Returns PA_ERR_ARG for null
 * pointers, H_q % H_kv != 0, negative window or hints, misalignment, an
 * unknown dtype, a missing or non-finite scale of an FP8 operand;
 * PA_ERR_UNSUPPORTED for head_dim not in {64,128,256} or a block size outside
 * the set above; PA_ERR_WORKSPACE when split-K partials are needed and the
 * workspace is too small; PA_ERR_CUDA when a launch fails.
 *
 * With both hints set the call only enqueues kernels, so it can be recorded
 * by a CUDA stream capture and replayed from a graph (replays read the
 * buffers' current contents); the work-list schedule is the exception.  The first call on a device sets kernel
 * attributes and queries occupancy; make it before capturing.
 */
int pa_decode(void *dst, const void *q, const void *kCache, const void *vCache,
              const int32_t *blockTables, const int32_t *seqLens,
              const int32_t *queryLens, float scale, int window, int kvBlockSize,
              const pa_params *params, void *stream);

/*
 * pa_workspace_size -- bytes of workspace pa_decode needs for these params
 * (split-K partial maxima/sums and outputs for max(1, P) partitions, the
 * allocation rule aiter PR #2914's review asks for).  Uses the hints; with a
 * zero span hint it assumes the longest row fills max_blocks_per_seq blocks,
 * with a zero query-length hint it assumes one query token per row (size the
 * workspace from real hints when rows carry several query tokens).
 * Returns 0 when the call is one-shot; (size_t)-1 on invalid params.  The
 * workspace needs no initialisation.
 * Host only; needs a CUDA device only when num_sms is not fixed (it queries
 * the current device's SM count and occupancy).
 */
size_t pa_workspace_size(const pa_params *params, int kvBlockSize);

/*
 * pa_plan -- the dispatcher's decision for these params, without launching.
 * num_sms / ctas_per_sm: 0 queries the current device; > 0 fixes them
 * (host-only use, e.g. on a machine without a GPU).  Host only.
 */
int pa_plan(const pa_params *params, int kvBlockSize, int num_sms, int ctas_per_sm,
            pa_plan_info *out);

/*
 * pa_visible_ranges -- the [lo, hi) each query token sees (section "What
 * changes" of the gllm page: max(0, end - window) .. end), computed on the
 * device with the same span function the kernels use.
 *   lo, hi       device int32 [sum(queryLens)], packed in batch order
 *   seqLens, queryLens, windows (may be NULL)  device int32 [batch]
 * Returns PA_ERR_ARG for null outputs/lengths, batch < 0 or window < 0.
 */
int pa_visible_ranges(int32_t *lo, int32_t *hi, const int32_t *seqLens,
                      const int32_t *queryLens, int window, const int32_t *windows,
                      int batch, void *stream);

/*
 * pa_unreachable_blocks -- for every row, how many leading KV blocks no query
 * token of this call or of any later call can see again.  With window w > 0
 * a token at position p sees p-w+1 .. p, and later tokens sit at larger
 * positions, so every block that ends at or before the row's earliest
 * visible position, max(0, S-L+1-w), is dead: floor(that / kvBlockSize)
 * blocks.  With w = 0 nothing is dead.  The cache still holds them; a
 * caller's block allocator may free (and reuse) those blocks (gllm PR #116,
 * "What changes": freeing blocks a window can no longer reach is left to a
 * separate change).  Rows with queryLens[b] = 0 report 0.
 *   count        device int32 [batch] (output)
 *   seqLens, queryLens, windows (may be NULL)  device int32 [batch]
 * Returns PA_ERR_ARG for null pointers, batch < 0 or window < 0, and
 * PA_ERR_UNSUPPORTED for a block size outside [16, 1024] or not a power of two.
 */
int pa_unreachable_blocks(int32_t *count, const int32_t *seqLens, const int32_t *queryLens,
                          int window, const int32_t *windows, int kvBlockSize, int batch,
                          void *stream);

/*
 * pa_decode_host -- end-to-end call with host buffers: copies q, blockTables,
 * seqLens, queryLens (and windows) from host memory into the caller's
 * workspace, runs pa_decode, copies dst back, and synchronises the stream.
 * The KV caches stay on the device (they are resident state).  Host buffers
 * should be pinned: a pinned buffer that is mapped into the current context
 * (CUDA's default for pinned memory under unified addressing) is read in
 * place by one staging kernel for all inputs, and a mapped, 16-byte aligned
 * dst_host is written in place by the kernels, so no copy engine is used
 * for it; other (pageable, unmapped) buffers are moved with
 * cudaMemcpyAsync.  The library checks with the driver that each buffer
 * lies inside one pinned allocation before reading or writing it in place.
 * All host buffers must stay valid and unmodified until the call returns.
 *   dst_host          host bf16 [sum(queryLens)][H_q][head_dim]
 *   q_host            host bf16 or FP8 codes (q_dtype), same shape
 *   blockTables_host, seqLens_host, queryLens_host  host int32
 *   params->windows   host int32 [batch] or NULL (host memory in this call)
 *   params->workspace device, >= pa_host_workspace_size() bytes
 * Hints are computed from the host lengths and need not be set.
 */
int pa_decode_host(void *dst_host, const void *q_host, const void *kCache,
                   const void *vCache, const int32_t *blockTables_host,
                   const int32_t *seqLens_host, const int32_t *queryLens_host,
                   float scale, int window, int kvBlockSize, const pa_params *params,
                   void *stream);

/* Workspace bytes pa_decode_host needs (staging for q, dst and the tables,
 * plus the split-K workspace); (size_t)-1 on invalid params. */
size_t pa_host_workspace_size(const pa_params *params, int kvBlockSize, int window,
                              const int32_t *seqLens_host, const int32_t *queryLens_host);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device
 * memory.  (The pages have no counterpart: this is a library convenience.)
 *
 * pa_decode needs a caller-allocated workspace for its split-K partials.
 * Callers that cannot call cudaMalloc -- code running under another
 * framework's allocator, plugins handed only input and output buffers, hot
 * paths that must not allocate -- use this entry point instead: the partials
 * live in a static device array compiled into the library,
 * PA_NOALLOC_SCRATCH_BYTES (32 MiB) per GPU, which every GPU that loads the
 * library holds until the process exits.  Arguments are those of pa_decode;
 * params->workspace and workspace_bytes are ignored.  The caller still
 * passes every input and output.
 *
 *  - The first call on a device looks up the array's device address with
 *    that device current; make it before any stream capture.  A reset device
 *    (cudaDeviceReset) has a new context and a new array: the first call
 *    after the reset looks the address up again, so make that one before
 *    any capture as well.
 *  - All calls on a device share the array: calls whose kernels overlap on
 *    the GPU race.  Nothing in it needs to start at zero; each call reads
 *    only partials it wrote itself.
 *  - A call whose partials need more than PA_NOALLOC_SCRATCH_BYTES returns
 *    PA_ERR_WORKSPACE before launching anything (pa_last_error() gives the
 *    bytes needed); tight hints keep the need small.  PA_ERR_CUDA if the
 *    array's address cannot be obtained.
 *  - It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define PA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

int pa_decode_noalloc(void *dst, const void *q, const void *kCache, const void *vCache,
                      const int32_t *blockTables, const int32_t *seqLens,
                      const int32_t *queryLens, float scale, int window, int kvBlockSize,
                      const pa_params *params, void *stream);

/*
 * pa_extents_host -- the two hints pa_params takes, from host copies of the
 * lengths: *max_span = longest union span over rows with queryLen > 0 (the
 * row's visible positions [max(0, S-L+1-window), S) for window > 0, else
 * [0, S)), *max_query_len = longest queryLen.  windows may be NULL (scalar
 * window).  Returns PA_ERR_ARG on a row with queryLen > seqLen or a negative
 * length or window.  Host only.
 */
int pa_extents_host(const int32_t *seqLens, const int32_t *queryLens,
                    const int32_t *windows, int window, int batch, int *max_span,
                    int *max_query_len);

/* Reads the device status word (PA_DEV_* bits) of the current device into
 * *status and clears it when clear != 0.  Synchronises the stream. */
int pa_device_status(unsigned int *status, int clear, void *stream);

/* Message of the last error on this thread ("" after success). */
const char *pa_last_error(void);

/* Library version string. */
const char *pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H */
