/*
 * eagleattn.h -- C ABI of libeagleattn: EAGLE-3 mixed joint-softmax attention
 * on NVIDIA B200 (sm_100a).
 *
 * The operation (NeMo AutoModel API page "eagle.ring_attention", class
 * _CachedRingAttention, class docstring): each query row t attends, in ONE
 * softmax, to
 *   - block 0: the sequence keys/values cache_k[:,0] / cache_v[:,0], causally
 *     (key position <= query position, the diagonal included), optionally
 *     restricted to the packed document of the row (page "eagle.ulysses_attention",
 *     _block0_forward, parameter cu_seqlens), with global positions
 *     q_pos_offset + t and k_pos_offset + s (page "target_cp",
 *     attach_cp_kv_gather_hooks: local queries against gathered keys under a
 *     global causal mask);
 *   - every block i >= 1: one per-position "diagonal" logit
 *     (Q_t . K_i_t) * scale with value V_i_t.
 * Everything is combined through the online-softmax log-sum-exp merge
 * (page "eagle.ring_attention", _update_out_and_lse and _merge_diag).  The
 * backward applies the FlashAttention identity against the MERGED out/lse and
 * adds the diagonal gradients in closed form (same class docstring; page
 * "eagle.zigzag_ring_attention", zigzag_ring_flash_attn_varlen_backward).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers (cudaMalloc'd or equivalent)
 *     unless stated otherwise.  The caller owns every buffer; the library
 *     allocates no tensor memory.  Its only persistent device state is one
 *     4-byte status word per device, created by the first call on that device.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls enqueue work and return without synchronising.
 *   - Layouts (FlashAttention style, element strides, head stride = D,
 *     innermost stride = 1):
 *       q, out, grad_out, dq      [B, Tq, H, D]       strides (q_stride_b, q_stride_t, D, 1)
 *       cache_k, cache_v, dk, dv  [B, NB, Tk, H, D]   strides (kv_stride_b, kv_stride_blk,
 *                                                              kv_stride_t, D, 1)
 *       lse                       [B, H, Tq] fp32, natural log, CONTIGUOUS (page
 *                                 "eagle.ulysses_attention", _gather_lse: the kernel
 *                                 reads lse with fixed strides)
 *       cu_seqlens                int32 [num_docs + 1], device, global positions
 *   - Return value: EAGLE_ATTN_OK (0) or a negative eagle_attn_status.  Host-side
 *     argument errors are detected before anything is enqueued.  Problems only
 *     the device can see (malformed cu_seqlens) make the kernels skip their
 *     work and set the device status word; read it with eagle_attn_get_status()
 *     after synchronising.  No kernel traps or asserts.
 */
#ifndef EAGLEATTN_H
#define EAGLEATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Version of this ABI.  The params struct is versioned and read by field
 * name, never by position (cf. page "eagle.ring_attention",
 * require_flash_attn_version: positional binding across releases silently
 * binds arguments to the wrong slots). */
#define EAGLE_ATTN_ABI_VERSION 4

typedef enum eagle_attn_status {
    EAGLE_ATTN_OK = 0,
    EAGLE_ATTN_ERR_NULL = -1,        /* a required pointer is NULL */
    EAGLE_ATTN_ERR_ABI = -2,         /* abi_version or struct_size mismatch */
    EAGLE_ATTN_ERR_DTYPE = -3,       /* unsupported dtype / out_dtype combination */
    EAGLE_ATTN_ERR_SHAPE = -4,       /* bad B/Tq/Tk/H/D/num_blocks */
    EAGLE_ATTN_ERR_STRIDE = -5,      /* strides overlap or are not representable */
    EAGLE_ATTN_ERR_ALIGN = -6,       /* pointer or row not 16-byte aligned */
    EAGLE_ATTN_ERR_VARLEN = -7,      /* cu_seqlens given with B != 1, or num_docs < 1 */
    EAGLE_ATTN_ERR_WORKSPACE = -8,   /* workspace NULL or smaller than required */
    EAGLE_ATTN_ERR_UNSUPPORTED = -9, /* a valid request no kernel here serves */
    EAGLE_ATTN_ERR_CUDA = -10,       /* a CUDA runtime call failed */
    EAGLE_ATTN_ERR_DEVICE = -11,     /* device-side check failed (see eagle_attn_get_status) */
    EAGLE_ATTN_ERR_SCRATCH_LIMIT = -12 /* eagle_attn_bwd_noalloc: problem needs more scratch than
                                          EAGLE_ATTN_NOALLOC_SCRATCH_BYTES */
} eagle_attn_status;

/* Device-side status codes (eagle_attn_get_status). */
#define EAGLE_ATTN_DEV_OK 0
#define EAGLE_ATTN_DEV_BAD_CU_SEQLENS 1   /* cu_seqlens[0] != 0 or not non-decreasing */
#define EAGLE_ATTN_DEV_DOC_TOO_LONG 2     /* a document is longer than max_seqlen */
#define EAGLE_ATTN_DEV_POS_OUTSIDE 3      /* a query or key position lies past cu_seqlens[num_docs] */
#define EAGLE_ATTN_DEV_TIMEOUT 4          /* a pipeline wait gave up (a library bug; no input causes it) */
#define EAGLE_ATTN_DEV_BAD_TILE 5         /* a q_tiles / q_tile_rows entry out of range, misaligned or out of order */
#define EAGLE_ATTN_DEV_SMEM_ALIGN 6       /* dynamic shared memory not 1024-byte aligned (a library bug) */

typedef enum eagle_attn_dtype {
    EAGLE_ATTN_F32 = 0,
    EAGLE_ATTN_BF16 = 1
} eagle_attn_dtype;

/* How eagle_attn_bwd delivers dq, dk, dv. */
typedef enum eagle_attn_grad_mode {
    EAGLE_ATTN_GRAD_STORE = 0,          /* written in `dtype` (default) */
    EAGLE_ATTN_GRAD_ACCUMULATE_F32 = 1  /* fp32 buffers (same element strides), the call's
                                           gradient ADDED to what they hold: the chunked
                                           schedule sums the key-chunk contributions of a
                                           query chunk and the query-chunk contributions of
                                           a key chunk this way.  Tensor-core path only. */
} eagle_attn_grad_mode;

typedef enum eagle_attn_impl {
    EAGLE_ATTN_IMPL_AUTO = 0,        /* tensor-core path when it applies, else generic */
    EAGLE_ATTN_IMPL_TENSOR_CORE = 1, /* tcgen05/TMEM/TMA kernels; bf16, D in {64, 128} */
    EAGLE_ATTN_IMPL_GENERIC = 2      /* CUDA-core kernels; f32 or bf16, D <= 128 */
} eagle_attn_impl;

typedef struct eagle_attn_params {
    uint32_t struct_size;      /* = sizeof(eagle_attn_params) */
    uint32_t abi_version;      /* = EAGLE_ATTN_ABI_VERSION */

    int32_t dtype;             /* eagle_attn_dtype of q, cache_k, cache_v, grad_out, dq, dk, dv */
    int32_t out_dtype;         /* dtype of out: = dtype, or EAGLE_ATTN_F32 (partial blocks to merge) */
    int32_t impl;              /* eagle_attn_impl */

    int32_t B, Tq, Tk, H, D;   /* Tk = block-0 key length; num_blocks > 1 requires Tk == Tq */
    int32_t num_blocks;        /* NB >= 1: block 0 + (NB - 1) diagonal blocks */
    int32_t causal;            /* 1: key position <= query position (default); 0: no position mask */
    int32_t deterministic;     /* backward, tensor-core path: 0 (default) = one dK/dV/dQ kernel,
                                  five products per tile pair, dQ summed with fp32 atomics (the
                                  order of the additions, so the last bits of dq, vary from run
                                  to run); 1 = bitwise reproducible: a dK/dV kernel and a dQ
                                  kernel (which recomputes S and dP), no atomics.  The CUDA-core
                                  path is always reproducible. */
    float scale;               /* softmax scale (typically D^-0.5) */
    int64_t q_pos_offset;      /* global position of query row 0 */
    int64_t k_pos_offset;      /* global position of block-0 key 0 */

    const int32_t *cu_seqlens; /* device int32 [num_docs + 1] or NULL; requires B == 1 */
    int32_t num_docs;
    int32_t max_seqlen;        /* longest document; checked on the device */

    int64_t q_stride_b, q_stride_t;                     /* elements; q, out, grad_out, dq */
    int64_t kv_stride_b, kv_stride_blk, kv_stride_t;    /* elements; cache_k, cache_v, dk, dv */

    const void *q;
    const void *cache_k;
    const void *cache_v;
    void *out;                 /* forward output; backward input (the MERGED out) */
    float *lse;                /* forward output; backward input (the MERGED lse) */

    const void *grad_out;      /* backward only */
    void *dq, *dk, *dv;        /* backward outputs (dtype); dk/dv cover all NB blocks */
    void *workspace;           /* backward scratch, >= eagle_attn_bwd_workspace_size() bytes */
    size_t workspace_bytes;

    /* Optional profiling hook: cudaEvent_t handles (as void*) recorded on the
     * call's stream immediately before and after the call's main attention
     * kernel (the block-0 kernel of eagle_attn_fwd / eagle_attn_bwd).  NULL =
     * not recorded. */
    void *prof_start;
    void *prof_stop;

    int32_t grad_mode;         /* eagle_attn_grad_mode (backward) */

    /* Tensor-core path: optional device int32 list of num_q_tiles query row
     * starts.  Without q_tile_rows each is a multiple of 128 in [0, Tq) and names
     * a 128-row tile (rows past Tq ignored).  The forward computes exactly those
     * tiles, one CTA each in list order, and leaves every other row of out and
     * lse untouched: one launch serves an emulated rank's rows of a chunk
     * schedule, its key chunks merged inside the kernel.  A bad entry raises
     * EAGLE_ATTN_DEV_BAD_TILE and that tile is skipped.  NULL = all rows. */
    const int32_t *q_tiles;
    int32_t num_q_tiles;

    /* ABI 4.  Optional device int32 list of num_q_tiles row counts, 1 .. 128, one
     * per q_tiles entry: entry i then names rows [q_tiles[i], q_tiles[i] +
     * q_tile_rows[i]) with no alignment (start + rows <= Tq), so segments of
     * documents of any length can be listed (page "eagle.zigzag_ring_attention",
     * get_half_index: a rank's front and back half of every document).
     *   Forward: computes exactly those rows, one CTA per entry.
     *   Backward (tensor-core path, deterministic = 0; q_tiles with or without
     *   q_tile_rows): entries sorted by start and disjoint; the gradients of the
     *   loss through exactly those rows' outputs -- dq of those rows (the other
     *   rows of dq untouched) and their contributions to dk, dv (block 0, and the
     *   diagonal blocks of those rows; the other rows of the diagonal blocks
     *   untouched).  With EAGLE_ATTN_GRAD_ACCUMULATE_F32, one call per emulated
     *   rank sums a chunk schedule's backward.  A list out of range or out of
     *   order raises EAGLE_ATTN_DEV_BAD_TILE (entries out of range are skipped).
     * NULL = whole 128-row tiles as above. */
    const int32_t *q_tile_rows;
} eagle_attn_params;

/* Returns EAGLE_ATTN_ABI_VERSION of the loaded library. */
int eagle_attn_abi_version(void);

/* Fills *p with defaults: struct_size, abi_version, dtype = out_dtype = BF16,
 * impl = AUTO, causal = 1, offsets 0, deterministic 0, all pointers NULL,
 * strides 0 (0 = contiguous, derived from the shape). */
void eagle_attn_params_init(eagle_attn_params *p);

/*
 * Forward.  Reads q, cache_k, cache_v (+ cu_seqlens); writes out [B,Tq,H,D]
 * (out_dtype) and lse [B,H,Tq] (fp32, natural log).  A row with no visible
 * key and no diagonal block gets lse = -inf and out = 0.
 * Pages: "eagle.ring_attention" _fa_forward (returns (out, lse[B,H,S])) and
 * _CachedRingAttention; "eagle.ulysses_attention" _block0_forward.
 */
int eagle_attn_fwd(const eagle_attn_params *p, void *stream);

/* Bytes of workspace eagle_attn_bwd needs for *p (0 on invalid params). */
size_t eagle_attn_bwd_workspace_size(const eagle_attn_params *p);

/*
 * Backward.  Reads q, cache_k, cache_v, out and lse (both MERGED, as written
 * by eagle_attn_fwd or by a merge chain), grad_out; writes dq [B,Tq,H,D] and
 * dk, dv [B,NB,Tk,H,D] (all blocks).  Uses the caller's workspace.
 * Pages: "eagle.ulysses_attention" _block0_backward (FlashAttention backward
 * against the merged out/lse); "eagle.ring_attention" _CachedRingAttention
 * (diagonal grads in closed form).
 */
int eagle_attn_bwd(const eagle_attn_params *p, void *stream);

/*
 * eagle_attn_bwd_noalloc -- the backward of eagle_attn_bwd for callers that
 * cannot allocate device memory.  (The NeMo AutoModel pages have no
 * counterpart; this is a service of this library.)
 *
 * Who needs it: code that may not call cudaMalloc and has no workspace to
 * hand over -- for example a plugin running inside a host framework that owns
 * every byte of device memory and exposes no workspace hook, or a latency-
 * critical loop that must not call cudaMalloc because it can synchronise the
 * device.  Such callers still pass every input and output buffer; only the
 * backward's scratch (the fp32 dQ accumulator and the per-row D_t, the bytes
 * eagle_attn_bwd_workspace_size() reports) comes from the library.
 *
 * Where the scratch lives: one static device array of
 * EAGLE_ATTN_NOALLOC_SCRATCH_BYTES (32 MiB) inside the library.  Every GPU on
 * which the library's kernels are loaded holds those 32 MiB until the process
 * exits.  The first call on a device looks up the array's device address for
 * that device (cudaGetSymbolAddress, with that device current) and caches it;
 * make that first call before any stream capture.  No call allocates or frees
 * memory (no cudaMalloc, no cudaFree, no allocating library routine).
 *
 * Limits and sharing: problems whose scratch exceeds the array (at D = 128,
 * B*Tq*H above about 65,000 rows) are rejected with
 * EAGLE_ATTN_ERR_SCRATCH_LIMIT before anything is enqueued; use
 * eagle_attn_bwd with a workspace for those.  Every call on a device shares the
 * same array and leaves its contents behind; the call clears what must start
 * at zero itself.  Calls whose kernels overlap on the GPU (on different
 * streams without ordering between them) race on the array and give wrong
 * gradients: order them.
 *
 * Arguments, layouts and results are those of eagle_attn_bwd; p->workspace and
 * p->workspace_bytes are ignored.
 */
#define EAGLE_ATTN_NOALLOC_SCRATCH_BYTES (32u << 20)
int eagle_attn_bwd_noalloc(const eagle_attn_params *p, void *stream);

/*
 * Online-softmax merge of a block into a running state, in place:
 *   lse' = log(exp(lse) + exp(block_lse)),
 *   out' = exp(lse - lse') * out + exp(block_lse - lse') * block_out.
 * out: fp32 [B,T,H,D] contiguous; lse, block_lse: fp32 [B,H,T] contiguous;
 * block_out: [B,T,H,D] contiguous in block_dtype (F32 or BF16).
 * init != 0 copies the block into the state instead (_init_out_and_lse).
 * lse = -inf marks an empty part; two empty parts stay (-inf, 0) with no NaN.
 * D must be 64 or 128, B and H at most 65535, T at most 65535 * 128
 * (EAGLE_ATTN_ERR_SHAPE otherwise).
 * Page "eagle.ring_attention", _update_out_and_lse / _init_out_and_lse;
 * page "eagle.zigzag_ring_attention", update_out_and_lse.
 */
int attn_merge_out_lse(float *out, float *lse, const void *block_out, int block_dtype,
                       const float *block_lse, int B, int T, int H, int D, int init,
                       void *stream);

/*
 * Merge the diagonal blocks 1..num_blocks-1 of *p into the running state
 * (p->out as fp32 [B,Tq,H,D] with q's strides, p->lse [B,H,Tq]): for each row
 * the block's lse is the single logit (Q_t . K_i_t) * scale and its out is
 * V_i_t.  p->out_dtype must be EAGLE_ATTN_F32.  Requires Tk == Tq.
 * Page "eagle.ring_attention", _merge_diag.
 */
int attn_merge_diag(const eagle_attn_params *p, void *stream);

/* dst[i] = (dst_dtype) src[i] for i < count (fp32 running out -> q dtype;
 * page "eagle.ulysses_attention", cached_ulysses_attention returns q's dtype).
 * src and dst need only their element alignment (4 bytes; 2 for a bf16 dst):
 * 16-byte aligned pairs take the vector path, others (row ranges of an lse,
 * say) an element-wise one.  EAGLE_ATTN_ERR_ALIGN otherwise. */
int attn_finalize(const float *src, void *dst, int dst_dtype, size_t count, void *stream);

/* Reads the status word of the current device (synchronous copy; call after
 * synchronising the streams that ran kernels).  *code = EAGLE_ATTN_DEV_*. */
int eagle_attn_get_status(int *code);
/* Resets the status word of the current device to EAGLE_ATTN_DEV_OK. */
int eagle_attn_clear_status(void);

/* Number of kernels this library has launched in this process (all devices);
 * lets a caller count the launches inside a timed region. */
uint64_t eagle_attn_launch_count(void);

/* Self-test of the failure path every pipeline wait in the tensor-core kernels
 * takes: one CTA waits, with the kernels' bounded wait and a limit of limit_ns
 * (1 .. 10^9), on an mbarrier that nothing arrives at.  The wait gives up, the
 * kernel raises EAGLE_ATTN_DEV_TIMEOUT in the device status word and returns;
 * the context stays usable.  Returns EAGLE_ATTN_ERR_SHAPE for a limit out of
 * range, else the launch status.  (No counterpart on the pages; a service of
 * this library for testing its own failure detection.) */
int eagle_attn_selftest_wait_timeout(int64_t limit_ns, void *stream);

/* Static, human-readable text for an eagle_attn_status value. */
const char *eagle_attn_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* EAGLEATTN_H */
