/*
 * dkv.h -- C ABI of libdkv: single-token decode attention (GQA/MHA, NeoX
 * RoPE) over a paged KV cache split between CPU-pinned host memory and GPU
 * HBM, for NVIDIA B200 (sm_100a).
 *
 * Method (DirectKV README, opening summary and Attribution; SplitKernel
 * README, Overview and Key Features): the KV cache of a sequence is split at
 * block granularity between host memory and device memory.  Host-resident
 * blocks are read by the GPU directly from mapped pinned memory into shared
 * memory, with no staging copy in HBM; device-resident blocks are read from
 * HBM.  Each side produces split-K partial results (an un-normalised
 * attention output and a log-sum-exp per query head and split), and a merge
 * combines all partials into the exact softmax attention output.
 *
 * Conventions shared by every entry point:
 *   - Every function returns DKV_OK (0) or a negative DKV_ERR_* code; the
 *     message of the last failure on the calling thread is available from
 *     dkv_last_error_string().  No function aborts or throws.
 *   - "device pointer": memory the GPU of the handle can read or write
 *     (cudaMalloc'd, or the device alias of mapped pinned host memory).
 *     "host pointer": ordinary CPU memory.
 *   - K/V element storage is 16-bit (IEEE binary16 or bfloat16), stored
 *     UN-ROTATED; the library applies RoPE to keys as it reads them.
 *   - Paged pool layout, for both pools: [num_blocks][Hkv][block_size][D],
 *     row-major; one (block, kv head) tile is block_size*D contiguous elements.
 *   - Logical positions: token t of a sequence is at position t; the query of
 *     a sequence of length L is at position L.
 *   - Query head hq reads KV head hq / G, G = Hq / Hkv (consecutive groups).
 */
#ifndef DKV_H
#define DKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DKV_API __attribute__((visibility("default")))
#else
#define DKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ------------------------------------------------------ */
#define DKV_OK 0
#define DKV_ERR_INVALID_ARG (-1) /* a pointer, size or enum is out of its documented range */
#define DKV_ERR_UNSUPPORTED (-2) /* valid request the library does not implement (head dim, group size) */
#define DKV_ERR_CUDA (-3)        /* a CUDA runtime call failed; see dkv_last_error_string() */
#define DKV_ERR_NO_MEMORY (-4)   /* device or pinned host allocation failed */

/* ---- device-side status bits (read with dkv_get_status) ----------------- */
#define DKV_STATUS_BAD_BLOCK_ID 1 /* a block table entry is outside both pools */
#define DKV_STATUS_BAD_SEQ_LEN 2  /* seq_lens[b] < 0 or beyond the table / handle capacity */
#define DKV_STATUS_COPY_TIMEOUT 4 /* a tile copy into shared memory did not complete within 2 s; the
                                     affected rows are NaN (the kernel stopped copying and returned) */
#define DKV_STATUS_INTERNAL 8     /* the HBM kernel found its shared memory misaligned and did nothing */

typedef enum { DKV_KV_F16 = 0, DKV_KV_BF16 = 1 } dkv_kv_dtype;

typedef struct dkv_config {
  int32_t num_q_heads;        /* Hq >= 1 */
  int32_t num_kv_heads;       /* 1 <= Hkv <= 4096, Hq % Hkv == 0; G = Hq/Hkv in {1, 2, 4} */
  int32_t head_dim;           /* D in {64, 128} */
  int32_t block_size;         /* S tokens per block: multiple of 16, 16 <= S <= 1024 */
  int32_t kv_dtype;           /* dkv_kv_dtype */
  double rope_base;           /* NeoX RoPE base; 0 disables rotation */
  double scale;               /* softmax scale; 0 means 1/sqrt(D) */
  int32_t max_batch;          /* largest batch passed to dkv_attn_decode */
  int32_t max_blocks_per_seq; /* largest number of blocks of one sequence */
  int32_t device;             /* CUDA device ordinal the handle is bound to */
  int32_t host_ctas;          /* CTAs of the zero-copy host kernel; 0 = chosen per call:
                                 16 while the host pool holds at least 1/50 of the device
                                 pool's blocks (the host stream carries the step), else 8
                                 (the HBM kernel beside it keeps more of its speed) */
} dkv_config;

typedef struct dkv_handle dkv_handle;
typedef struct CUstream_st* dkv_stream_t; /* the same type as cudaStream_t; NULL = legacy default stream */

/*
 * dkv_create -- validate cfg and allocate the per-handle workspace on
 * cfg->device: the split-K partial buffers, the device status word, two work
 * counters per split launch, the per-pool block lists, an auxiliary
 * high-priority stream and two events used to fork/join the host and HBM
 * kernels.  The partial buffers hold 2 * (16 * 8 * SMs + G * max_batch * Hkv)
 * rows of head_dim + 1 floats (about 20 MB for 148 SMs, head_dim 128), enough
 * for one split-K unit per warp of a full wave with up to 16 query rows each;
 * the block lists take 8 * max_batch * max_blocks_per_seq bytes.  On success
 * *out owns all of it until dkv_destroy.
 * Errors: INVALID_ARG (null pointers, out-of-range fields), UNSUPPORTED
 * (head_dim or group size), NO_MEMORY, CUDA.
 */
DKV_API int dkv_create(const dkv_config* cfg, dkv_handle** out);

/* dkv_destroy -- synchronise the handle's streams and free everything it owns.
 * NULL is accepted and ignored. */
DKV_API int dkv_destroy(dkv_handle* h);

/*
 * dkv_attn_decode -- one decode-attention step for a batch of sequences.
 *
 *   q            device, fp32 [batch][Hq][D]: the new token's query, un-rotated;
 *                8-byte aligned.  All four pool pointers must be 16-byte aligned.
 *   k_host,v_host  device aliases of MAPPED pinned host memory (see
 *                dkv_host_pool_alloc), pool layout, >= host_split blocks.
 *                May be NULL only when host_split == 0.
 *   k_dev,v_dev  device memory (HBM), pool layout, >= num_dev_blocks blocks.
 *                May be NULL only when num_dev_blocks == 0.
 *   block_table  device, int32 [batch][block_table_stride]: entry j of row b
 *                is the physical id of logical block j (tokens j*S .. j*S+S-1)
 *                of sequence b.  Ids in [0, host_split) index the host pool;
 *                ids in [host_split, host_split + num_dev_blocks) index the
 *                device pool at id - host_split.  Only entries
 *                j < ceil(seq_lens[b]/S) are read.
 *   seq_lens     device, int32 [batch]: context length L_b (tokens already in
 *                the cache; the new token's own K/V are not part of it).
 *                0 <= L_b <= min(block_table_stride, max_blocks_per_seq) * S.
 *   out          device, fp32 [batch][Hq][D]: softmax attention output.
 *   stream       all work is ordered on this stream (forked internally onto
 *                the handle's auxiliary stream and joined back); the call
 *                neither allocates nor synchronises.  One call at a time per
 *                handle: calls that overlap on different streams race on the
 *                handle's workspace.
 * Host-side argument errors return INVALID_ARG / UNSUPPORTED before anything
 * is launched.  Table entries outside both pools and out-of-range lengths are
 * detected on the device: the status word records DKV_STATUS_* bits and the
 * affected rows of out are written as NaN (there is no device trap).
 */
DKV_API int dkv_attn_decode(dkv_handle* h, const float* q, const void* k_host, const void* v_host,
                    const void* k_dev, const void* v_dev, const int32_t* block_table,
                    const int32_t* seq_lens, int32_t host_split, float* out, dkv_stream_t stream,
                    int32_t batch, int32_t block_table_stride, int32_t num_dev_blocks);

/*
 * dkv_attn_decode_multi -- num_queries (Tq) query tokens per sequence over the
 * same split cache, for speculative verification or chunked prefill (the
 * pages' CUDA test runs a "Prefill (all new KV)" case, DirectKV README,
 * Step 6).  Query i of sequence b sits at position L_b + i and attends to the
 * cached tokens t < L_b + i, so the cache must already hold the tokens
 * L_b .. L_b + Tq - 2 (see dkv_append_kv) and the table must cover them.
 * Tq = 1 computes exactly what dkv_attn_decode computes.
 *   q    device fp32 [batch][Tq][Hq][D]        out  device fp32 [batch][Tq][Hq][D]
 *   Tq * (Hq / Hkv) <= 16 and batch * Tq <= max_batch; the rest as for
 *   dkv_attn_decode (L_b + Tq - 1 <= table capacity, else status + NaN rows).
 * Both contractions run on the tensor cores (mma.sync, with 16-bit hi + lo
 * splits of the rotated keys, the queries and the softmax weights).
 * Errors: as dkv_attn_decode. */
DKV_API int dkv_attn_decode_multi(dkv_handle* h, int32_t num_queries, const float* q, const void* k_host,
                                  const void* v_host, const void* k_dev, const void* v_dev,
                                  const int32_t* block_table, const int32_t* seq_lens, int32_t host_split,
                                  float* out, dkv_stream_t stream, int32_t batch, int32_t block_table_stride,
                                  int32_t num_dev_blocks);

/*
 * dkv_attn_decode_staged -- the staged-prefetch comparator: the design the
 * zero-copy method is measured against (SplitKernel README, Overview:
 * prefetch-based offloading that first moves offloaded data back into HBM;
 * DirectKV README, Artifact Evaluation: the Pie / FlexGen prefetch baselines).
 * The first host_split blocks of the host pools are copied into the device
 * staging pools k_stage / v_stage with cudaMemcpyAsync (copy engine, pinned
 * host -> HBM) on `stream`, then both pools are read by the HBM split-K
 * kernel and merged.  Same arguments and results as dkv_attn_decode, plus:
 *   k_stage, v_stage  device memory (HBM) of >= host_split blocks each, pool
 *                     layout, 16-byte aligned; owned by the caller.
 * It costs host_split blocks of HBM and one HBM write + read of them per call;
 * dkv_attn_decode needs neither.  Errors: as dkv_attn_decode. */
DKV_API int dkv_attn_decode_staged(dkv_handle* h, const float* q, const void* k_host, const void* v_host,
                                   const void* k_dev, const void* v_dev, const int32_t* block_table,
                                   const int32_t* seq_lens, int32_t host_split, float* out, dkv_stream_t stream,
                                   int32_t batch, int32_t block_table_stride, int32_t num_dev_blocks, void* k_stage,
                                   void* v_stage);

/*
 * dkv_append_kv -- write side of the cache: project the new token of every
 * sequence to K and V and store them, un-rotated, at its position (DirectKV
 * README, opening summary: the fused kernel includes the K/V projection of new
 * tokens; Step 6 checks K and V of "all new KV").
 *   x           device fp32 [batch][hidden]: hidden state of the new token
 *   w_k, w_v    device 16-bit (the handle's kv_dtype) [Hkv*D][hidden] row-major;
 *               row h*D + d produces dim d of kv head h
 *   hidden      > 0, multiple of 8; x, w_k, w_v and the pools 16-byte aligned
 *   block_table, seq_lens, host_split, num_dev_blocks, pools: as for
 *               dkv_attn_decode.  The new token goes to position L = seq_lens[b]
 *               (the cache holds L tokens): block table entry L / S must name
 *               its block, row L % S of that block is written.  seq_lens is not
 *               changed; the caller advances it.
 * k = W_k x and v = W_v x are accumulated in fp32 and rounded to the 16-bit
 * type (nearest, ties to even).  Host-resident blocks are written through the
 * mapped pointer.  Async on `stream`; positions beyond the table or ids
 * outside both pools set DKV_STATUS_* bits and skip the store.
 * Errors: INVALID_ARG, CUDA. */
DKV_API int dkv_append_kv(dkv_handle* h, const float* x, const void* w_k, const void* w_v, int32_t hidden,
                          const int32_t* block_table, const int32_t* seq_lens, int32_t host_split, void* k_host,
                          void* v_host, void* k_dev, void* v_dev, dkv_stream_t stream, int32_t batch,
                          int32_t block_table_stride, int32_t num_dev_blocks);

/* dkv_get_status -- synchronise the handle's device, return the accumulated
 * DKV_STATUS_* bits in *status and clear them. */
DKV_API int dkv_get_status(dkv_handle* h, int32_t* status);

/* dkv_last_error_string -- message of the last failed call on this thread
 * ("" if none).  The string stays valid until the next failing call. */
DKV_API const char* dkv_last_error_string(void);

/* dkv_last_launch_count -- number of kernels the handle's last successful
 * dkv_attn_decode launched: with blocks in both pools the pool-lists kernel,
 * the zero-copy host kernel, the HBM split-K kernel and the merge (4); with
 * one pool, that pool's split kernel and the merge (2). */
DKV_API int dkv_last_launch_count(const dkv_handle* h, int32_t* count);

/* dkv_query_plan -- the split-K decomposition of the HBM kernel of a
 * dkv_attn_decode call whose blocks all sit in HBM, for (batch,
 * block_table_stride): splits per sequence and blocks per split.  The plan
 * aims at one unit (sequence, split, kv head) per resident warp of the
 * kernel; with 2 or more sequences, at 2 units per warp when every unit still
 * holds at least 1024 tokens (finer units keep ragged batches balanced).
 * With host blocks as well, each launch splits the list of its own pool's
 * blocks of every sequence, and the HBM launch plans for the warps left beside
 * the zero-copy host kernel: one unit per warp while the host part carries the
 * step, two (under the same conditions as above) when the host pool holds
 * less than 1/50 of the device pool's blocks. */
DKV_API int dkv_query_plan(const dkv_handle* h, int32_t batch, int32_t block_table_stride, int32_t* num_splits,
                   int32_t* blocks_per_split);

/* ---- decode without any allocation ---------------------------------------
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory or keep a handle: a serving engine that
 * hands all GPU memory to its own allocator at start-up (a library cudaMalloc
 * would then fail or upset its accounting), a latency-critical loop in which
 * cudaMalloc/cudaFree may synchronise the device, or a plugin behind a plain
 * C interface that only sees raw pointers on each call.
 *
 * dkv_attn_decode_noalloc -- the same computation as dkv_attn_decode, with
 * the configuration passed per call and no handle.  It allocates nothing:
 * its scratch (status word, work counters, RoPE frequencies, per-pool block
 * lists, split partials) is one fixed array of DKV_NOALLOC_SCRATCH_BYTES
 * compiled into the library, held on every GPU that loads the library until
 * the process exits.
 *   cfg          read for this call only; cfg->max_batch is ignored, the
 *                other fields mean what they mean for dkv_create.
 *   status_out   device int32 or NULL: receives the DKV_STATUS_* bits of
 *                this call (the scratch status word is cleared at its start).
 *   other arguments as for dkv_attn_decode.  All kernels run in order on
 *   `stream` (the host-stream and HBM kernels do not overlap here): a small
 *   set-up kernel (frequencies, cleared status and counters), with blocks in
 *   both pools the pool-lists kernel, the split kernel of each pool and the
 *   merge -- one launch more than dkv_attn_decode.
 * The first call on a device looks up the device address of the scratch
 * array (cudaGetSymbolAddress) and sets the kernels' shared-memory limits;
 * make that first call before any stream capture.  Every call on a device
 * shares the one array and finds the previous call's contents in it, so calls
 * that may overlap on the GPU (other streams, other threads) race: order them.
 * The number of splits is cut down until the partials fit; a batch for which
 * even one split per pool in use cannot fit (batch * num_q_heads beyond about
 * DKV_NOALLOC_SCRATCH_BYTES / (4 * (head_dim + 1) * pools in use), less 8
 * bytes per table block of every sequence when both pools hold blocks) is
 * rejected with DKV_ERR_INVALID_ARG before anything is launched.  No cudaMalloc, cudaFree
 * or other allocating call is made. */
#define DKV_NOALLOC_SCRATCH_BYTES (16u << 20)
DKV_API int dkv_attn_decode_noalloc(const dkv_config* cfg, const float* q, const void* k_host, const void* v_host,
                                    const void* k_dev, const void* v_dev, const int32_t* block_table,
                                    const int32_t* seq_lens, int32_t host_split, float* out, int32_t* status_out,
                                    dkv_stream_t stream, int32_t batch, int32_t block_table_stride,
                                    int32_t num_dev_blocks);

/* ---- allocation-failure injection (test only) ----------------------------
 * dkv_debug_fail_alloc -- TEST ONLY: makes the nth device allocation (1-based)
 * of the next dkv_create on the calling thread fail as if the GPU were out of
 * memory; 0 disarms.  The hook is cleared by the first dkv_create that
 * reaches its allocations, whether or not it failed.  Lets tests check that
 * a failed create returns DKV_ERR_NO_MEMORY, frees what it had allocated and
 * leaves the device usable, without exhausting real GPU memory.  dkv_create
 * makes 7 device allocations.  Errors: INVALID_ARG (nth < 0). */
DKV_API int dkv_debug_fail_alloc(int32_t nth);

/* dkv_debug_stall_copy -- TEST ONLY: in the next dkv_attn_decode on the
 * calling thread whose HBM kernel moves its tiles with tensor copies (a call
 * with blocks in both pools, where that kernel runs beside the zero-copy host
 * kernel), the warp that takes that kernel's first work unit arms the
 * barrier of the unit's first tile copy but issues no copy, so its bounded
 * wait runs out (about 2 s): the call must then report
 * DKV_STATUS_COPY_TIMEOUT, write NaN for that warp's units and leave the
 * device usable.  The hook is
 * cleared by that call; 0 disarms it.  Always returns DKV_OK. */
DKV_API int dkv_debug_stall_copy(int32_t enable);

/* ---- RoPE check (test only) ----------------------------------------------
 * dkv_debug_rope -- TEST ONLY: applies NeoX RoPE exactly as the decode
 * kernels do, so that the rotation can be compared element by element with an
 * exact reference at large positions (DirectKV README, opening summary: the
 * attention kernel applies "Neox RoPE rotation" to the keys it loads).  One
 * warp walks the key tiles in order, as a decode warp walks the tiles of its
 * units: the same lane layout, fp64-reduced seed angles, 4-position fp32
 * recurrence and chaining rule (a tile that starts 16 positions after the
 * previous one continues the rotation state; at most 16 tiles share one
 * seed).  Queries are rotated by the decode kernels' query path with a scale
 * of 1.  The frequencies are base^(-2i/head_dim), computed as dkv_create does.
 *   k         device 16-bit (kv_dtype) [num_tiles][16][head_dim] un-rotated key
 *             rows, 16-byte aligned; row r of tile i sits at position tile_pos[i] + r
 *   tile_pos  device int32 [num_tiles], each >= 0
 *   k_out     device fp32 [num_tiles][16][head_dim]: the rotated rows
 *   q, q_pos, q_out  device fp32 [num_q][head_dim], int32 [num_q], fp32 [num_q][head_dim]
 *   rope_base > 1; head_dim 64 or 128; k_out, q and q_out 8-byte aligned.
 * Async on `stream`; allocates nothing.  Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
DKV_API int dkv_debug_rope(int32_t kv_dtype, int32_t head_dim, double rope_base, const void* k,
                           const int32_t* tile_pos, int32_t num_tiles, float* k_out, const float* q,
                           const int32_t* q_pos, int32_t num_q, float* q_out, dkv_stream_t stream);

/* ---- per-kernel timing ---------------------------------------------------
 * dkv_profile_begin -- record CUDA events around every kernel of the next
 * max_calls dkv_attn_decode calls, each on the stream that kernel runs on
 * (the host-stream kernel runs on the handle's auxiliary stream).  Events are
 * created here, never inside dkv_attn_decode.  Not for use while a stream is
 * being captured into a CUDA graph.  Errors: INVALID_ARG, CUDA. */
DKV_API int dkv_profile_begin(dkv_handle* h, int32_t max_calls);

/* dkv_profile_timeline -- synchronise the handle's device and return, for
 * recorded call number `call` (0 = the first after dkv_profile_begin), the
 * start and stop of each kernel in t_ms[6] = {host start, host stop, HBM
 * start, HBM stop, merge start, merge stop}, in ms from the earliest start
 * among them; -1 for a kernel that did not run.  Shows whether the host-stream
 * and HBM kernels overlapped.  Call it before dkv_profile_end.  Errors:
 * INVALID_ARG (no kernel of that call recorded), CUDA. */
DKV_API int dkv_profile_timeline(dkv_handle* h, int32_t call, float* t_ms);

/* dkv_profile_end -- synchronise the handle's device, then return in ms[k] the
 * summed device time of kernel k over the recorded calls and in counts[k] how
 * many launches were recorded: k = 0 zero-copy host kernel, 1 HBM split-K
 * kernel, 2 LSE merge.  Releases the events.  Errors: INVALID_ARG, CUDA. */
DKV_API int dkv_profile_end(dkv_handle* h, float* ms, int32_t* counts);

/* ---- host KV pool ------------------------------------------------------- */

/* dkv_host_pool_alloc -- page-locked host memory that is mapped into the
 * address space of every GPU (cudaHostAlloc Mapped|Portable).  *ptr is both
 * the host address and, with unified addressing, the device alias to pass as
 * k_host / v_host.  Release with dkv_host_pool_free.  Errors: INVALID_ARG,
 * NO_MEMORY. */
DKV_API int dkv_host_pool_alloc(size_t bytes, void** ptr);
DKV_API int dkv_host_pool_free(void* ptr);

/* ---- partitioner (host side, setup only) --------------------------------
 * Placement of logical blocks between the host pool and the device pool
 * (SplitKernel README, Key Features: host/device KV cache partitioning and
 * placement / offloading-ratio utilities). */
typedef enum {
  DKV_PLACE_PREFIX_HOST = 0, /* the oldest round(f*n_b) blocks of each sequence on the host, the newest on HBM */
  DKV_PLACE_RANDOM = 1       /* round(f*n_b) blocks of each sequence chosen uniformly at random for the host */
} dkv_placement;

typedef struct dkv_plan_params {
  int32_t block_size;   /* S, as in dkv_config */
  int32_t placement;    /* dkv_placement */
  double host_fraction; /* f in [0, 1] */
  int32_t shuffle_ids;  /* nonzero: physical ids are a random permutation within each pool */
  uint64_t seed;        /* seeds the splitmix64 stream used for random choices */
} dkv_plan_params;

typedef struct dkv_plan_result {
  int32_t host_split;     /* number of host blocks; host ids are [0, host_split) */
  int32_t num_dev_blocks; /* device ids are [host_split, host_split + num_dev_blocks) */
  int64_t host_tokens;    /* valid tokens placed in host blocks */
  int64_t dev_tokens;     /* valid tokens placed in device blocks */
} dkv_plan_result;

/*
 * dkv_plan_blocks -- build a block table for sequences of the given lengths.
 *   seq_lens     host, int32 [batch]
 *   block_table  host, int32 [batch][block_table_stride], written; entries
 *                past ceil(L_b/S) are set to -1.
 * Host blocks are numbered first (sequence-major, then logical order), then
 * device blocks, before the optional shuffle.  Deterministic for a seed.
 * Errors: INVALID_ARG (null pointers, f outside [0,1], a sequence that needs
 * more than block_table_stride blocks, more than 2^31-1 blocks in total).
 */
DKV_API int dkv_plan_blocks(const dkv_plan_params* params, const int32_t* seq_lens, int32_t batch, int32_t* block_table,
                    int32_t block_table_stride, dkv_plan_result* result);

/*
 * dkv_plan_offload -- choose the host fraction of the KV cache (SplitKernel
 * README, Key Features: placement / offloading-ratio utilities; DirectKV
 * README, Figure mapping, Fig 11b: GPU memory freed at long context).
 * With X = total KV bytes, the modelled step time of a placement with host
 * fraction f > 0 is T(f) = max(f*X / host_gbs, (1-f)*X / hbm_gbs): the
 * zero-copy host stream and the HBM kernel run concurrently and the slower one
 * sets the step.  T falls while the HBM side dominates and rises once PCIe
 * does, so the best such fraction is f* = host_gbs / (host_gbs + hbm_gbs),
 * with T(f*) = X / (host_gbs + hbm_gbs).  At f = 0 the HBM kernel runs alone,
 * T(0) = X / hbm_alone_gbs, which can be shorter: a kernel beside the host
 * stream is slower than alone.  An HBM budget for the cache forces
 * f >= 1 - budget/X.  The plan is f = 0 when the budget allows it and
 * T(0) <= T(f*); otherwise f = max(f*, that bound), capped at 1.
 *   kv_bytes        X > 0
 *   host_gbs        measured host read bandwidth of the host kernel (> 0)
 *   hbm_gbs         measured HBM read bandwidth of the HBM kernel while the
 *                   host kernel runs beside it (> 0)
 *   hbm_budget_bytes  HBM bytes the cache may occupy; < 0 means unlimited
 *   hbm_alone_gbs   measured HBM read bandwidth of the HBM kernel alone;
 *                   <= 0 if unknown (then f = 0 is never chosen)
 * Out: host_fraction, predicted step seconds, HBM bytes freed (f*X) and the
 * time-optimal fraction without a budget (0 or f*).  Pure host arithmetic;
 * errors: INVALID_ARG (sizes or rates not positive and finite, a NaN budget,
 * a non-finite hbm_alone_gbs). */
typedef struct dkv_offload_plan {
  double host_fraction;
  double step_seconds;
  double hbm_bytes_freed;
  double time_optimal_fraction;
} dkv_offload_plan;

DKV_API int dkv_plan_offload(double kv_bytes, double host_gbs, double hbm_gbs, double hbm_budget_bytes,
                             double hbm_alone_gbs, dkv_offload_plan* plan);

/*
 * dkv_pack_kv -- write logical K/V into the paged pools following a table.
 *   k_logical, v_logical  host, 16-bit [batch][Hkv][lmax][D]
 *   seq_lens, block_table host, as in dkv_plan_blocks
 *   k_host, v_host        host addresses of the host pool (>= host_split blocks)
 *   k_dev_stage, v_dev_stage  host staging copies of the device pool
 *                         (>= num_dev_blocks blocks) that the caller then
 *                         copies to HBM; may be NULL when num_dev_blocks == 0.
 * Token rows of a block past L_b are zeroed.  Errors: INVALID_ARG.
 */
DKV_API int dkv_pack_kv(const uint16_t* k_logical, const uint16_t* v_logical, int64_t lmax, const int32_t* seq_lens,
                int32_t batch, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                const int32_t* block_table, int32_t block_table_stride, int32_t host_split,
                int32_t num_dev_blocks, uint16_t* k_host, uint16_t* v_host, uint16_t* k_dev_stage,
                uint16_t* v_dev_stage);

#ifdef __cplusplus
}
#endif

#endif /* DKV_H */
