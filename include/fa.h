/*
 * fa.h -- C ABI of the B200 (sm_100a) decode / small-Q attention library
 * (libfa_b200.so).
 *
 * Operation (every entry point that computes):
 *
 *   O = softmax(Q K^T * scale) V
 *
 *   "SmallQ FlashAttention for Ascend 910B", section "接口" (interface):
 *   O = softmax(Q·Kᵀ/√headDim)·V on fp16 inputs with fp32 accumulation;
 *   the MXFlashAttn README (section "前向算子 API") gives the FlashAttention
 *   style forward calls flash_attn_func / flash_attn_with_kvcache with
 *   causal=True, GQA ratios 2/4/8 and head_dim 64/128 in fp16 and bf16;
 *   the same README's M1 kernel is a split-KV decode kernel.
 *
 * Conventions shared by all calls
 *   - Tensors are described by fa_tensor: a DEVICE pointer, an element type,
 *     a 4-D shape in [B, L, H, D] order and element strides.  The last
 *     dimension (D) must be contiguous (stride 1); the other strides are free,
 *     so a [H, L, D] buffer is passed as shape [1, L, H, D] with strides
 *     {H*L*D, D, L*D, 1}.  Base pointers must be 16-byte aligned and every
 *     stride a multiple of 8 elements (16 bytes).
 *   - q is [B, Lq, Hq, Dqk]; k is [B, Lk, Hkv, Dqk]; v is [B, Lk, Hkv, Dv];
 *     o is [B, Lq, Hq, Dv] of the same element type; Hq = g * Hkv (GQA:
 *     query head hq reads kv head hq / g).  Head dims: Dqk and Dv each any
 *     multiple of 8 from 8 to 256 (the SmallQ kernel's "任意 headDim" in
 *     "SmallQ FlashAttention for Ascend 910B", section "支持范围", within the
 *     16-byte stride rule above); a call runs on the compiled kernel whose
 *     dims cover it -- (64, 64), (128, 128), (192, 128) or (256, 256) -- with
 *     the extra dims read as zeros and never written.  Other dims return
 *     FA_ERR_UNSUPPORTED.  q, k, v and o share one type: FA_F16 or FA_BF16.
 *   - lse, when not NULL, is a DEVICE fp32 array [B, Hq, Lq] (contiguous)
 *     receiving the natural-log log-sum-exp of each row's scaled scores.
 *   - causal != 0 applies a causal mask aligned to the bottom-right corner:
 *     key j is visible to query i iff j <= i + n - Lq, n being the number of
 *     keys of that batch.  A row with no visible key gets O = 0, lse = -inf.
 *   - scale <= 0 selects 1/sqrt(Dqk).
 *   - num_splits <= 0 lets the library choose how the key range is split
 *     across CTAs; num_splits > 0 asks for about that many splits per
 *     (batch, kv-head, row block) unit (the result does not depend on it
 *     beyond fp32 rounding).
 *   - workspace: caller-owned DEVICE scratch of at least the size the
 *     matching *_workspace_size call returns (it may be NULL when that size
 *     is 0), 256-byte aligned; nothing in it needs initialising.  Calls that
 *     share a workspace must not overlap in time.  The library never
 *     allocates device memory and never synchronises the stream in the
 *     compute calls.
 *   - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *     All work is enqueued asynchronously on it; the caller keeps the
 *     buffers alive until it completes.
 *   - Errors: argument problems are detected on the host, before any launch,
 *     and returned as FA_ERR_INVALID_ARG / FA_ERR_UNSUPPORTED /
 *     FA_ERR_WORKSPACE with a message in fa_last_error(); a failed launch
 *     returns FA_ERR_CUDA.  No call silently falls back to a slower path.
 *
 * Thread safety: the compute calls may be issued from several host threads;
 * fa_last_error() and fa_last_dispatch() report the calling thread's last call.
 *
 * Device state: the library keeps, per device, the address of its status
 * word (fa_check_status) and of the allocation-free call's scratch array,
 * looked up on first use and cached for the life of the process.  A
 * cudaDeviceReset (or any other end of the device's primary context) makes
 * them stale: do not call the library on that device afterwards.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fa_status {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1, /* malformed shapes, strides, pointers or types */
    FA_ERR_UNSUPPORTED = 2, /* well-formed but outside the supported set */
    FA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required */
    FA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
    FA_ERR_TIMEOUT = 5      /* a kernel gave up waiting on its copy pipeline */
} fa_status;

typedef enum fa_dtype { FA_F16 = 0, FA_BF16 = 1 } fa_dtype;

/* A strided 4-D device tensor in [B, L, H, D] order (element strides). */
typedef struct fa_tensor {
    void *data;
    int32_t dtype; /* fa_dtype */
    int32_t reserved;
    int64_t shape[4];
    int64_t stride[4];
} fa_tensor;

/* Which kernels the calling thread's last compute call launched. */
typedef enum fa_variant {
    FA_VARIANT_AUTO = 0,
    FA_VARIANT_MMA = 1,     /* split-KV kernel, mma.sync tensor-core products */
    FA_VARIANT_SCALAR = 2,  /* split-KV kernel, fp32 FMA products (one packed row) */
    FA_VARIANT_TCGEN05 = 3, /* dense kernel on tcgen05 + TMEM (>= 128 packed rows, head dims 64/64, 128/128, 192/128) */
    FA_VARIANT_TCGEN05_SPLIT = 4 /* split-KV kernel on tcgen05 + TMEM: row blocks of 16 / 32 / 64 packed rows */
} fa_variant;

typedef struct fa_dispatch_info {
    int32_t variant;          /* fa_variant of the main kernel */
    int32_t grid;             /* CTAs launched for the main kernel */
    int32_t block;            /* threads per CTA of the main kernel */
    int32_t smem_bytes;       /* dynamic shared memory per CTA */
    int32_t tile_keys;        /* keys per pipeline stage */
    int32_t stages;           /* pipeline depth */
    int32_t rows_per_cta;     /* packed query rows per CTA (g * Lq packing) */
    int32_t units;            /* (batch, kv-head, row-block) work units */
    int32_t min_share_tiles;  /* least tiles a CTA is given */
    int32_t combine_launched; /* 1 if the LSE combine kernel was launched */
    int64_t work_tiles;       /* total key tiles (known on the host for fa_fwd; -1 for kvcache) */
    int32_t tcgen05_form;     /* fa_tcgen05_form of the tcgen05 kernel (0 for the other variants) */
    int32_t reserved;
} fa_dispatch_info;

/*
 * fa_fwd -- forward attention over dense Q/K/V (flash_attn_func).
 * q, k, v, o as in the conventions above (Lk taken from k->shape[1]).
 */
FA_API fa_status fa_fwd(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, fa_tensor *o,
                 float *lse, int causal, float scale, int num_splits, void *workspace,
                 size_t workspace_bytes, void *stream);

/*
 * fa_fwd_workspace_size -- bytes of workspace fa_fwd needs for these shapes
 * on the current device (0 when no key range is split between CTAs).  The
 * first half of the two-phase call of "SmallQ FlashAttention for Ascend
 * 910B", section "aclnn API 调用": a GetWorkspaceSize call sizes the scratch,
 * the caller allocates it, then the compute call runs on the caller's
 * stream.  Host only (no launch, no allocation); the arguments are those of
 * the matching compute call (o and data pointers are not read).
 */
FA_API fa_status fa_fwd_workspace_size(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v,
                                int causal, int num_splits, size_t *bytes);

/*
 * fa_decode_kvcache -- attention of new queries against a dense KV cache
 * (flash_attn_with_kvcache).  k_cache/v_cache are [B, Lmax, Hkv, D]; batch b
 * attends to its first cache_seqlens[b] keys (0 <= cache_seqlens[b] <= Lmax,
 * a DEVICE int32 array [B]; slots at and beyond cache_seqlens[b] are never
 * used and may hold anything, NaN included).  causal/scale as above with
 * n = cache_seqlens[b].
 */
FA_API fa_status fa_decode_kvcache(const fa_tensor *q, const fa_tensor *k_cache, const fa_tensor *v_cache,
                            const int32_t *cache_seqlens, fa_tensor *o, float *lse, int num_splits,
                            int causal, float scale, void *workspace, size_t workspace_bytes,
                            void *stream);

/*
 * fa_decode_kvcache_workspace_size -- bytes of workspace fa_decode_kvcache
 * needs for these shapes on the current device: the GetWorkspaceSize phase
 * of the aclnn two-phase call ("SmallQ FlashAttention for Ascend 910B",
 * section "aclnn API 调用"), as for fa_fwd_workspace_size.  The size does not
 * depend on the cache lengths (they live on the device).
 */
FA_API fa_status fa_decode_kvcache_workspace_size(const fa_tensor *q, const fa_tensor *k_cache,
                                           const fa_tensor *v_cache, int num_splits,
                                           size_t *bytes);

/*
 * fa_decode_kvcache_paged -- fa_decode_kvcache over a paged K/V cache.
 *
 * The M1 kernel of the MXFlashAttn README is a "split-KV paged decode"
 * kernel, and the README's capability table ("能力矩阵", the dense / varlen /
 * paged KV cache row) lists paged KV caches as implemented.  The pages do not
 * spell out the page layout; this call takes the FlashAttention block-table
 * convention that the README's flash_attn_with_kvcache interface implies:
 *   k_pages  [num_blocks, page, Hkv, Dqk], v_pages [num_blocks, page, Hkv, Dv]
 *            (fa_tensor, shape[0] = num_blocks, shape[1] = page: a power of
 *            two from 16 to 2^20; last dim contiguous, 16-byte aligned);
 *   block_table  DEVICE int32, batch b's entries at
 *            block_table[b * block_table_stride + i], i < max_blocks_per_seq;
 *   key j of batch b (j < cache_seqlens[b]) is row j % page of block
 *   block_table[b * block_table_stride + j / page].
 * Everything else (q, o, lse, causal, scale, num_splits, workspace, stream)
 * is as for fa_decode_kvcache; cache_seqlens[b] is clamped to
 * [0, max_blocks_per_seq * page].  Blocks may be shared or in any order.
 * Table entries for pages past a batch's length are never used for values
 * (they may hold anything); an entry outside [0, num_blocks) inside the
 * length reads as zeros.  The caller owns every buffer; nothing is allocated
 * and nothing is synchronised.
 */
FA_API fa_status fa_decode_kvcache_paged(const fa_tensor *q, const fa_tensor *k_pages, const fa_tensor *v_pages,
                                         const int32_t *block_table, int64_t block_table_stride,
                                         int max_blocks_per_seq, const int32_t *cache_seqlens, fa_tensor *o,
                                         float *lse, int num_splits, int causal, float scale, void *workspace,
                                         size_t workspace_bytes, void *stream);

/* Bytes of workspace fa_decode_kvcache_paged needs for these shapes on the current device. */
FA_API fa_status fa_decode_kvcache_paged_workspace_size(const fa_tensor *q, const fa_tensor *k_pages,
                                                        const fa_tensor *v_pages, int max_blocks_per_seq,
                                                        int num_splits, size_t *bytes);

/*
 * fa_decode_kvcache_append -- append new tokens' K / V to the cache, then
 * attend (the order of flash_attn_with_kvcache with new k / v, the interface
 * the MXFlashAttn README follows; its capability table lists paged KV append
 * among the verified cases).
 *   k_new [B, Lnew, Hkv, Dqk], v_new [B, Lnew, Hkv, Dv]: DEVICE, q's type.
 *   k_cache / v_cache: dense [B, Lmax, Hkv, D] when block_table is NULL,
 *   else paged [num_blocks, page, Hkv, D] with block_table /
 *   block_table_stride / max_blocks_per_seq as for fa_decode_kvcache_paged.
 *   Token t of batch b is written to cache position cache_seqlens[b] + t
 *   (dense row, or row pos % page of block block_table[b, pos / page]); a
 *   position at or past the capacity, or an invalid block number, is not
 *   written.  The attention then sees cache_seqlens[b] + Lnew keys (clamped
 *   to the capacity); cache_seqlens itself is not modified.  With causal,
 *   query i (of Lq, normally Lq = Lnew) sees keys j <= i + n - Lq.
 * Everything else is as for fa_decode_kvcache; the workspace is the size
 * fa_decode_kvcache_workspace_size (dense) or
 * fa_decode_kvcache_paged_workspace_size (paged) returns.  The copy runs as
 * its own small kernel ahead of the attention kernels, on the same stream.
 */
FA_API fa_status fa_decode_kvcache_append(const fa_tensor *q, const fa_tensor *k_new, const fa_tensor *v_new,
                                          fa_tensor *k_cache, fa_tensor *v_cache, const int32_t *block_table,
                                          int64_t block_table_stride, int max_blocks_per_seq,
                                          const int32_t *cache_seqlens, fa_tensor *o, float *lse, int num_splits,
                                          int causal, float scale, void *workspace, size_t workspace_bytes,
                                          void *stream);

/*
 * fa_fwd_varlen -- fa_fwd over packed variable-length sequences.
 *
 * The MXFlashAttn README's public entry points include
 * flash_attn_varlen_func, and the CSDN "FlashAttention on Ascend CANN" post
 * lists packed (not padded) variable-length input among the operator's
 * features; the layout is FlashAttention's cu_seqlens convention:
 *   q [1, total_q, Hq, Dqk], k [1, total_k, Hkv, Dqk], v [1, total_k, Hkv, Dv],
 *   o [1, total_q, Hq, Dv] (fa_tensor, shape[0] = 1);
 *   cu_seqlens_q / cu_seqlens_k: DEVICE int32 [batch + 1], non-decreasing,
 *   cu[0] = 0; sequence b owns query tokens [cu_q[b], cu_q[b+1]) and key
 *   tokens [cu_k[b], cu_k[b+1]);
 *   max_seqlen_q / max_seqlen_k: bounds on the lengths (rows and keys beyond
 *   them are not computed / not read);
 *   lse, when not NULL: DEVICE fp32 [Hq, total_q] (contiguous).
 * Attention runs within each sequence: query i of sequence b attends its own
 * keys, with the causal mask aligned to the bottom-right corner of that
 * sequence (key j visible iff j <= i + n_b - Lq_b); a sequence with no keys
 * gives O = 0, lse = -inf.  scale, num_splits, workspace (size from
 * fa_fwd_varlen_workspace_size), stream and errors as for fa_fwd.
 */
FA_API fa_status fa_fwd_varlen(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v,
                               const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int batch,
                               int max_seqlen_q, int max_seqlen_k, fa_tensor *o, float *lse, int causal, float scale,
                               int num_splits, void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace fa_fwd_varlen needs for these shapes on the current device. */
FA_API fa_status fa_fwd_varlen_workspace_size(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, int batch,
                                              int max_seqlen_q, int max_seqlen_k, int num_splits, size_t *bytes);

/*
 * fa_decode_kvcache_noalloc -- fa_decode_kvcache for callers that cannot
 * allocate device memory (for example a plugin inside a serving runtime that
 * owns all device memory and forbids allocation after start-up, or a decode
 * loop that cannot afford the implicit synchronisation cudaMalloc may cause).
 * The pages have no counterpart to this call; it exists for such callers.
 * Same arguments and results as fa_decode_kvcache minus the workspace: the
 * split-KV scratch is a fixed array of fa_noalloc_scratch_bytes() bytes
 * (8 MiB) compiled into the library, held on every GPU that loads it until
 * the process exits.  Shapes (or num_splits) needing more scratch than that
 * are rejected with FA_ERR_UNSUPPORTED and a message; nothing is allocated,
 * ever.  The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current: make that first call
 * before any stream capture.  All calls on a device share the array and it
 * keeps the last call's contents (nothing in it needs to start at zero), so
 * calls whose GPU work overlaps -- on different streams or from racing host
 * threads -- race on it and must be serialised by the caller.  The array's
 * address is cached per device for the life of the process (as is the
 * status word's, see fa_check_status): after cudaDeviceReset, or anything
 * else that destroys the device's primary context, both are stale and this
 * library must not be called again in that process.
 */
FA_API fa_status fa_decode_kvcache_noalloc(const fa_tensor *q, const fa_tensor *k_cache,
                                           const fa_tensor *v_cache, const int32_t *cache_seqlens,
                                           fa_tensor *o, float *lse, int num_splits, int causal,
                                           float scale, void *stream);

/* Size in bytes of the fixed scratch array fa_decode_kvcache_noalloc uses. */
FA_API size_t fa_noalloc_scratch_bytes(void);

/*
 * fa_check_status -- this library's own addition; the pages have no
 * counterpart (their calls report errors only through return codes).
 * Synchronises `stream`, then reports whether any kernel of this library on
 * the current device gave up waiting on its copy pipeline since the last
 * check (FA_ERR_TIMEOUT) and clears that record.  FA_ERR_CUDA if the stream
 * itself reports an error.  The record is ONE word per device, shared by
 * every stream and host thread: a check on one stream also reads (and
 * clears) a timeout recorded by a kernel that another stream or thread
 * launched, so a caller that must attribute a timeout to one stream has to
 * serialise its checks with the other users of the device.
 */
FA_API fa_status fa_check_status(void *stream);

/* Message of the calling thread's last failed call ("" after success). */
FA_API const char *fa_last_error(void);

/*
 * fa_last_dispatch -- what the calling thread's last successful compute call
 * launched (kernel variant, grid, split partition, whether the combine ran):
 * the counterpart of get_last_dispatch_info() in the MXFlashAttn README
 * (section "前向算子 API"), which reports the backend that served the last
 * forward call.  Host only; the record is per host thread.
 */
FA_API void fa_last_dispatch(fa_dispatch_info *info);

/*
 * Tuning / test hook: force the main-kernel variant for later calls of this
 * process (FA_VARIANT_AUTO restores the library's choice).
 *   FA_VARIANT_MMA     tensor cores (mma.sync m16n8k16, keys as the 16-row
 *                      side, up to 8 packed query rows as the 8-column side);
 *   FA_VARIANT_SCALAR  fp32 FMA dot products, one packed query row only
 *                      (g * Lq == 1), the "scalar fp32 dot product" form of
 *                      "SmallQ FlashAttention for Ascend 910B", section
 *                      "算法要点".
 *   FA_VARIANT_TCGEN05 the 5th-gen tensor cores (tcgen05.mma, S, P and O in
 *                      TMEM) on blocks of 128 or 256 packed query rows (see
 *                      fa_tcgen05_form), whole key range per CTA, no split
 *                      and no combine; dense fa_fwd calls with head dims
 *                      64/64, 128/128 or 192/128.
 *   FA_VARIANT_TCGEN05_SPLIT  the split-KV kernel on the 5th-gen tensor
 *                      cores: a unit is a block of up to 64 packed query rows
 *                      (16, 32 or 64: the g * Lq rows of a GQA group with
 *                      their speculative positions), so K / V are streamed
 *                      once for all of them; S^T = K Q^T with the 128 keys of
 *                      a tile as the M side and the rows as N, O^T = V^T P^T,
 *                      both accumulated in TMEM; head dims up to 192 / 128
 *                      (every call API: dense, kvcache, paged, varlen, append).
 * The library's own choice: FA_VARIANT_TCGEN05 for dense fa_fwd calls with at
 * least 128 packed rows (g * Lq >= 128), head dims 64/64, 128/128 or 192/128
 * and at least 32 CTAs of rows (prefill-shaped calls); FA_VARIANT_TCGEN05_SPLIT for more than 8 packed
 * rows (g * Lq > 8) with Dqk <= 192 and Dv <= 128 once the K / V re-reads it
 * saves over blocks of 8 rows reach 128 MB (B * Lk * Hkv * (Dqk + Dv) * 2
 * bytes per block, Lk the cache capacity for the kvcache calls: below that its
 * higher fixed cost per call loses); FA_VARIANT_MMA otherwise --
 * measured on B200 it is faster than the FMA variant even for one packed row.
 * A forced variant that does not support the call's shapes makes the call
 * fail with FA_ERR_UNSUPPORTED.
 */
FA_API fa_status fa_force_variant(int variant);

/*
 * Forms of the tcgen05 kernel (all: 128 packed rows per query tile, 128-key
 * K / V tiles, accumulators in TMEM, the whole key range per CTA):
 *   FA_TCGEN05_ONE_TILE       retired (an earlier one-tile design whose
 *                             softmax warps issued the products; removed):
 *                             forcing it is FA_ERR_INVALID_ARG;
 *   FA_TCGEN05_TWO_TILES      two tiles per CTA and a dedicated MMA warp: one
 *                             tile's products run while the other tile's
 *                             softmax does (S single-buffered per tile);
 *   FA_TCGEN05_ONE_TILE_MMA   the two-tile kernel's pipeline with one tile, S
 *                             double-buffered.
 * The library's choice: two tiles when that still gives every SM a CTA
 * (ceil(R / 256) * Hkv * B >= SMs), else FA_TCGEN05_ONE_TILE_MMA.
 */
typedef enum {
    FA_TCGEN05_AUTO = 0,
    FA_TCGEN05_ONE_TILE = 1,
    FA_TCGEN05_TWO_TILES = 2,
    FA_TCGEN05_ONE_TILE_MMA = 3
} fa_tcgen05_form;

/* Tuning / test hook: force the tcgen05 kernel's form for later calls of this
 * process (FA_TCGEN05_AUTO restores the library's choice). */
FA_API fa_status fa_force_tcgen05_form(int form);

/*
 * Test hook for the failure path: the next compute call of this process
 * (split-KV or tcgen05 prefill kernel) bounds its pipeline waits by
 * wait_limit_ns (instead of 4 s) and its first CTA leaves its first pipeline
 * stage empty -- no copy, no arrival -- so that CTA's consumers give up after
 * wait_limit_ns, record
 * FA_ERR_TIMEOUT in the device status word and return (as do the producer,
 * after a bounded wait for its copies in flight).  The call's outputs are
 * then unspecified; fa_check_status reports the timeout and later calls run
 * normally.  FA_ERR_INVALID_ARG unless 0 < wait_limit_ns <= 4e9.
 */
FA_API fa_status fa_test_stall_next_call(unsigned long long wait_limit_ns);

/*
 * Profiling: while enabled, each compute call brackets its main kernel and
 * its combine kernel with CUDA events on the call's stream (and launches them
 * without programmatic overlap, so each event pair times one kernel alone).
 * Enabling clears earlier records; disabling keeps them for fa_profile_read.
 * Calls captured into a CUDA graph record their events as event-record nodes,
 * so each replay of the graph writes that call's record again.
 * fa_profile_read synchronises nothing: call it after the stream (or the
 * graph's replay) has completed; it returns the summed milliseconds and the
 * number of timed launches of each kernel.
 */
FA_API fa_status fa_profile_enable(int on);
FA_API fa_status fa_profile_read(double *main_ms, int64_t *main_launches, double *combine_ms,
                          int64_t *combine_launches);

/*
 * fa_schedule -- host-side copy of the work partition the kernels compute on
 * the device (no device access; for inspection and tests).  Work is counted
 * in key tiles of `tile_keys` keys (a power of two); a unit is (batch, block
 * of `rows_per_cta` packed query rows, kv head) -- 8 for the mma.sync
 * split-KV kernel, 16 / 32 / 64 for the tcgen05 one (fa_last_dispatch's
 * rows_per_cta says which a call used) -- ordered batch-major, then row
 * block, then kv head, and owns t = ceil(visible keys / tile_keys) tiles.  In
 * the partition a unit with t > 0 tiles occupies t + seg_cost positions (its
 * tiles first; seg_cost stands for the fixed cost of a unit: 1 for the
 * mma.sync kernel, 4 for the tcgen05 one).  The W positions of all units are
 * laid end to end and cut into ctas_used = min(num_ctas, ceil(W / min_share))
 * contiguous pieces, one per CTA, whose sizes differ by at most one position
 * (the first W mod ctas_used pieces are the longer ones); a piece that starts
 * in a unit's trailing positions starts with the next unit.  seqlens: HOST
 * int32 [B] (NULL: every batch has Lk keys).  For each of the first max_units
 * units the call writes its tile count and the first and last CTA whose piece
 * holds its tiles (-1, -1 for a unit with no tiles).  FA_ERR_INVALID_ARG for
 * inconsistent sizes (rows_per_cta must be in [1, 64], seg_cost in
 * [0, 1024]).
 */
FA_API fa_status fa_schedule(int B, int Lq, int Hq, int Hkv, int Lk, int causal, const int32_t *seqlens,
                             int num_ctas, int min_share, int tile_keys, int rows_per_cta, int seg_cost,
                             int64_t *work_tiles, int64_t *ctas_used, int32_t *unit_tiles,
                             int64_t *unit_first_cta, int64_t *unit_last_cta, int64_t max_units);

/* Kernels launched by this library in this process (both kinds). */
FA_API int64_t fa_launch_count(void);

/* Library version string. */
FA_API const char *fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
