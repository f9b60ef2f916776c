/*
 * paged_attn.h - C ABI of the B200 (sm_100a) paged KV-cache attention library.
 *
 * The library implements PagedAttention over a block-table KV cache as the
 * source pages describe it:
 *
 *   [P1] "Nano-vLLM-Ascend: lightweight LLM inference framework for Ascend NPU"
 *        section 2.1 (PageAttention memory management: 16-token blocks, the
 *        Block and BlockTable structures, per-block reference counts),
 *        section 2.2.1 (attention = softmax(q k^T / sqrt(d)) v),
 *        section 4.2 (the 1/sqrt(d) scale; reference counts checked for leaks).
 *   [P2] "Ascend NPU LLM inference optimisation: the vLLM-Ascend approach"
 *        section 2.1 (BlockAllocator over one pool), section 2.2 (PagedAttention
 *        operator: fill requests into fixed blocks, tile QK^T, softmax and V
 *        weighting), section 3.1 (256-byte aligned accesses; softmax in fp32),
 *        section 4 (block sharing for long contexts).
 *   [P3] "In-depth analysis of vllm-ascend: LLM inference architecture on
 *        Ascend hardware" section 1.1 / 3.1 (chunked prefill inside one device).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Device pointers are owned by the caller (e.g. PyTorch tensors).  The
 *   compute calls allocate no device memory and never synchronise the host;
 *   work is enqueued on `stream` (a cudaStream_t passed as void*, NULL = the
 *   legacy default stream).
 * - Every call returns a pa_status.  Arguments are validated on the host
 *   before anything is launched; a rejected call launches nothing and leaves
 *   all buffers untouched.  No call aborts or traps.
 * - Tensors are dense, row-major, in the layouts given per argument.
 * - Element type: PA_F16 (IEEE half) or PA_BF16 (bfloat16) for q, k, v, caches
 *   and out.  All softmax statistics and accumulators are fp32.
 * - KV cache layout (P1 s2.1, blocks stacked into one pool, P2 s2.1):
 *       cache[num_blocks][block_size][num_kv_heads][head_dim]
 *   separately for K and V.  Slot s = physical_block * block_size + row.
 * - block_tables: int32 [batch][max_blocks_per_seq]; entry j of row b is the
 *   physical block that holds tokens j*block_size .. j*block_size+block_size-1
 *   of sequence b; entries past ceil(context_lens[b]/block_size) are never read.
 * - context_lens: int32 [batch], tokens of each sequence INCLUDING any token
 *   written in this step.
 * - Supported: head_dim in {64, 128}; block_size in {16, 32, 64, 128, 256};
 *   num_q_heads a multiple of num_kv_heads with group size G = Hq/Hkv in
 *   {1, 2, 4, 8, 16}; query head h reads KV head h / G.
 * - Alignment (P2 s3.1): every tensor pointer must be 16-byte aligned.
 * - Device-resident indices (block table entries, slots, lengths) are trusted:
 *   the caller guarantees 0 <= entry < num_blocks, slot < num_blocks*block_size
 *   and context_lens[b] <= min(max_context_len, max_blocks_per_seq*block_size).
 *   Kernels that detect a broken device-side invariant record it in a device
 *   error word (pa_device_error) instead of trapping.
 */
#ifndef PAGED_ATTN_H
#define PAGED_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = -1,      /* null pointer, negative size, inconsistent shapes */
  PA_ERR_UNSUPPORTED = -2,  /* head_dim, block_size, group size or dtype outside the supported set */
  PA_ERR_ALIGN = -3,        /* a tensor pointer is not 16-byte aligned */
  PA_ERR_WORKSPACE = -4,    /* workspace missing or smaller than required */
  PA_ERR_CUDA = -5,         /* a CUDA runtime/driver call failed (launch error etc.) */
  PA_ERR_OOM = -6,          /* block pool has too few free blocks (state unchanged) */
  PA_ERR_NOT_FOUND = -7,    /* unknown sequence id / sequence already exists */
  PA_ERR_DEVICE = -8        /* a kernel recorded a broken device-side invariant */
} pa_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* pa_strerror(int status);

/* Library version as "major.minor.patch" (static string). */
const char* pa_version(void);

/* Asynchronous copy of `bytes` bytes from src to dst on `stream`            */
/* (cudaStream_t, NULL = legacy default stream), in whichever direction the  */
/* two addresses give (host, pinned host or device memory of the current     */
/* device; unified addressing decides).  Plumbing for callers that stage a   */
/* step's inputs into device memory without switching streams on their side:*/
/* it returns once the copy is queued; pinned host memory makes a host-side  */
/* copy asynchronous.  The caller keeps both buffers alive and unchanged     */
/* until the stream passes the copy.  bytes == 0 is a no-op; NULL dst or src */
/* with bytes > 0 -> PA_ERR_INVALID; a failed enqueue -> PA_ERR_CUDA.        */
int pa_copy_async(void* dst, const void* src, size_t bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* KV write (P1 s2.1 Block layout; P2 s2.2 "fill requests into fixed-size     */
/* blocks").                                                                  */
/*                                                                            */
/* For every t in [0, num_tokens) with slot_mapping[t] >= 0:                  */
/*   k_cache[slot / bs][slot % bs][h][:] = k[t][h][:]  (all h), same for v.   */
/* A bitwise copy (16-byte vectors); slot -1 means "skip this row".           */
/* k, v: [num_tokens][num_kv_heads][head_dim] device, read only.             */
/* slot_mapping: int64 [num_tokens] device.  Duplicate slots are undefined.  */
/* k_cache, v_cache: [num_blocks][block_size][num_kv_heads][head_dim] device.*/
/* k and v must not overlap the caches.  num_tokens == 0 is a no-op.         */
/* Launch: one kernel, with programmatic dependent launch.  It may start     */
/* while the preceding kernel on the stream finishes and waits for that     */
/* kernel to complete before it reads anything; a pa_decode after it may    */
/* start its set-up (reading context_lens and block_tables) before the      */
/* write completes, and waits for it before reading q or the cache.         */
/* ------------------------------------------------------------------------ */
int pa_write_kv(const void* k, const void* v, const int64_t* slot_mapping, int num_tokens,
                void* k_cache, void* v_cache, int num_blocks, int block_size, int num_kv_heads,
                int head_dim, int dtype, void* stream);

/* ------------------------------------------------------------------------ */
/* Block copy for copy-on-write (P1 s2.1 reference counts; P2 s4 block       */
/* sharing).  For each pair i: block pairs[2i+1] of both caches becomes a     */
/* bitwise copy of block pairs[2i].  pairs: int32 [num_pairs][2] device.     */
/* Source and destination blocks of all pairs must be distinct.             */
/* ------------------------------------------------------------------------ */
int pa_copy_blocks(const int32_t* pairs, int num_pairs, void* k_cache, void* v_cache, int num_blocks,
                   int block_size, int num_kv_heads, int head_dim, int dtype, void* stream);

/* ------------------------------------------------------------------------ */
/* Rotary position embedding fused with the KV write (P1 s3.1: each model    */
/* brings its rotary embedding; P1 s5.1: a rotary multiply of x by           */
/* per-position cos/sin tables, whose inverse negates sin; P2 s2.2: the      */
/* write into fixed-size blocks that follows it).                            */
/*                                                                            */
/* Pairing (rotate-half): element i of a head turns with element i + D/2 by  */
/* the angle of column i of the token's table row p = positions[t]:          */
/*   y[i]       = x[i] * cos[p][i] - x[i + D/2] * sin[p][i]                  */
/*   y[i + D/2] = x[i + D/2] * cos[p][i] + x[i] * sin[p][i]                  */
/* in fp32, rounded to nearest even.  For every token t:                     */
/*   q_out[t][h] = y(q[t][h])                    (all num_q_heads heads)     */
/* and, if slot = slot_mapping[t] >= 0 (slot -1: no cache write):            */
/*   k_cache[slot / bs][slot % bs][h] = y(k[t][h]),                          */
/*   v_cache[slot / bs][slot % bs][h] = v[t][h]  (bitwise)                   */
/* q, q_out: [num_tokens][num_q_heads][head_dim] device; q_out may equal q   */
/* (in place) but must not otherwise overlap any other argument.             */
/* k, v: [num_tokens][num_kv_heads][head_dim] device, read only.             */
/* positions, slot_mapping: int64 [num_tokens] device.                       */
/* cos_table, sin_table: fp32 [max_position][head_dim / 2] device, 16-byte   */
/* aligned, read only.  Caches as for pa_write_kv.  num_tokens == 0 is a     */
/* no-op (only the caches are checked).  num_tokens * (num_q_heads +         */
/* 3 * num_kv_heads) * head_dim / 16 must be below 2^31                      */
/* (PA_ERR_UNSUPPORTED otherwise).  A position outside [0, max_position)    */
/* leaves every row of that token unwritten and a slot >= num_blocks *       */
/* block_size leaves its cache rows unwritten; both set PA_ERRBIT_INDEX in   */
/* the device error word (pa_device_error).  One kernel launch, with       */
/* programmatic dependent launch (it waits for the preceding kernel before  */
/* it reads anything); a pa_decode that follows on the stream may start its */
/* set-up early and waits for this kernel before it reads q_out or the cache.*/
/* ------------------------------------------------------------------------ */
int pa_rope_write_kv(const void* q, void* q_out, const void* k, const void* v, const int64_t* positions,
                     const float* cos_table, const float* sin_table, int max_position,
                     const int64_t* slot_mapping, int num_tokens, int num_q_heads, void* k_cache,
                     void* v_cache, int num_blocks, int block_size, int num_kv_heads, int head_dim,
                     int dtype, void* stream);

/* ------------------------------------------------------------------------ */
/* Paged decode (P1 s2.2.1, s4.2; P2 s2.2, s3.1): one query token per        */
/* sequence attends to all context_lens[b] tokens of its sequence:           */
/*   out[b][h] = sum_t softmax_t(scale * <q[b][h], K_b[t][h/G]>) V_b[t][h/G] */
/* context_lens[b] == 0 gives out[b] = 0.                                    */
/*                                                                           */
/* Work split (split-K, P3 s3.1 read on one device): every (sequence, KV     */
/* head) is cut into 16-token chunks; all chunks, end to end, are shared out */
/* evenly over `grid` persistent CTAs.  The part of a sequence's context     */
/* that one CTA handles yields fp32 (max, sum, weighted V) in the workspace  */
/* unless it is the whole context; the CTA that finishes a context's last    */
/* part merges the parts by the log-sum-exp rule (atomic count, no waiting). */
/* One kernel is launched per call, with programmatic dependent launch: its */
/* set-up (reading context_lens and block_tables) may overlap the preceding */
/* kernel, and it waits for that kernel before reading q or the cache or    */
/* writing anything.  Once all of its loads are issued it lets the next     */
/* programmatically launched kernel on the stream (the next step's          */
/* pa_write_kv, or another decode) begin; that kernel waits for this one's  */
/* completion before touching memory.                                       */
/*                                                                           */
/* pa_decode_plan: the grid and workspace the call will use on the current   */
/* device.  num_partitions_or_0 > 0 fixes the number of CTAs (the number of  */
/* parts the chunk line is cut into); 0 fills the GPU (SMs x CTAs per SM).   */
/* max_pieces_out: partial slots of the workspace, batch*Hkv + grid.        */
/* max_context_len is only checked here (>= 0).  Output pointers may be NULL.*/
/* ------------------------------------------------------------------------ */
int pa_decode_plan(int batch, int num_q_heads, int num_kv_heads, int head_dim, int max_context_len,
                   int num_partitions_or_0, int* grid_out, int* max_pieces_out, size_t* workspace_bytes_out);

/* Bytes of device workspace pa_decode needs for these sizes (0 on bad args). */
size_t pa_decode_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                int max_context_len, int num_partitions_or_0);

/* q: [batch][num_q_heads][head_dim]; out: same shape; caches as above.      */
/* max_context_len: host-side upper bound of context_lens; block_tables rows */
/* must cover it (max_blocks_per_seq * block_size >= max_context_len).       */
/* workspace: device scratch of >= pa_decode_workspace_size() bytes, 256-byte */
/* aligned, owned by the caller.  It must be zero-filled before its first    */
/* use (its head holds per-context piece counters); every completed call     */
/* leaves those counters at zero again, so it needs no clearing afterwards   */
/* (a call that recorded PA_ERRBIT_TIMEOUT may leave them dirty: re-zero).  */
/* Two calls that run at the same time must use different workspaces.        */
int pa_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
              int max_blocks_per_seq, const int32_t* context_lens, int batch, int num_q_heads,
              int num_kv_heads, int head_dim, int block_size, int num_blocks, int max_context_len,
              float scale, int dtype, void* workspace, size_t workspace_bytes, int num_partitions_or_0,
              void* out, void* stream);

/* ------------------------------------------------------------------------ */
/* Cascade decode over shared prefixes (P1 s2.1: blocks carry reference     */
/* counts and forked sequences share their prefix blocks; P2 s4: block      */
/* sharing for long contexts).  Same result as pa_decode, but each shared   */
/* prefix block is read once for all sequences that share it:               */
/*   1. pa_decode's kernel over every sequence's private suffix, tokens     */
/*      seq_prefix_len[b] .. context_lens[b]-1, leaving (out, log-sum-exp);  */
/*   2. one pass over each group's shared prefix with the query rows of all */
/*      its members at once (head_dim 128: the CTA-pair tensor-core kernel   */
/*      of pa_prefill_chunk; head_dim 64: warp MMA), merged with step 1 by   */
/*      the log-sum-exp rule into out.                                      */
/* Groups: num_groups consecutive ranges of the batch, group g = sequences  */
/* group_start[g] .. group_start[g+1]-1 (int32 [num_groups+1], device,      */
/* non-decreasing); sequences outside every range, and groups whose prefix  */
/* is 0, get plain decode.  seq_prefix_len: int32 [batch], device: the      */
/* shared prefix length of each sequence's group (0 outside groups), a      */
/* multiple of 16, at most its context length; every member of a group     */
/* has the same value and maps its first seq_prefix_len/block_size block-   */
/* table entries to the same physical blocks (the prefix is read through    */
/* the group's first member).  max_group_size / max_prefix_len: host upper  */
/* bounds of group sizes and prefix lengths (they size the grid).           */
/* Workspace: pa_decode_cascade_workspace_size() bytes, 256-byte aligned,   */
/* zero-filled before first use; every completed call leaves its counters   */
/* at zero.  Two launches on `stream`; same argument checks and return      */
/* codes as pa_decode.  A prefix length that is not a multiple of 16 is     */
/* rounded down and sets PA_ERRBIT_INDEX.  At head_dim 128 step 2 is a      */
/* programmatic dependent launch: its CTAs may start in step 1's tail     */
/* (step 1 lets it launch only after the kernel before step 1 completed)   */
/* and read q, the tables and the prefix rows then; they wait for step 1   */
/* to complete before reading or writing out (no caller action needed).    */
/* ------------------------------------------------------------------------ */
size_t pa_decode_cascade_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                        int max_context_len, int num_partitions_or_0, int num_groups,
                                        int max_group_size, int max_prefix_len);
int pa_decode_cascade(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                      int max_blocks_per_seq, const int32_t* context_lens, int batch, int num_q_heads,
                      int num_kv_heads, int head_dim, int block_size, int num_blocks, int max_context_len,
                      float scale, int dtype, int num_groups, const int32_t* group_start,
                      const int32_t* seq_prefix_len, int max_group_size, int max_prefix_len, void* workspace,
                      size_t workspace_bytes, int num_partitions_or_0, void* out, void* stream);

/* ------------------------------------------------------------------------ */
/* Decode with library-owned scratch (no counterpart on the source pages).   */
/* Same computation, arguments and results as pa_decode, but without a      */
/* workspace argument: for callers that cannot allocate device memory where */
/* they run decode (inside CUDA graph capture, under a fixed memory pool,   */
/* or on a serving path that must not block on an allocation).  The scratch */
/* is one static device array of PA_DECODE_STATIC_SCRATCH_BYTES, reserved   */
/* on every GPU that loads the library until the process exits.  Calls that */
/* would need more (pa_decode_workspace_size() larger than that) return     */
/* PA_ERR_WORKSPACE.  Every other argument is checked as pa_decode checks  */
/* it, before anything is enqueued; a rejected call enqueues nothing.       */
/* Nothing is allocated: an accepted call clears the piece counters at the  */
/* head of the array (cudaMemsetAsync on `stream`) and runs the decode      */
/* kernel.  Because of that clear, decode on this entry point does not      */
/* start early under a preceding pa_write_kv / pa_rope_write_kv (pa_decode  */
/* does).  The first call on a device looks up the array's device address  */
/* (cudaGetSymbolAddress) with that device current; make that first call    */
/* before any stream capture.  All calls share the one array and it keeps   */
/* the last call's contents, so calls whose work overlaps on the GPU (other */
/* streams, other threads) race: serialise them.                            */
/* ------------------------------------------------------------------------ */
#define PA_DECODE_STATIC_SCRATCH_BYTES (8u << 20)
int pa_decode_static_scratch(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                             int max_blocks_per_seq, const int32_t* context_lens, int batch, int num_q_heads,
                             int num_kv_heads, int head_dim, int block_size, int num_blocks, int max_context_len,
                             float scale, int dtype, int num_partitions_or_0, void* out, void* stream);

/* ------------------------------------------------------------------------ */
/* INT8 KV cache (P1 s4.3: KV-cache compression and INT8 in the tuning      */
/* checklist; P2 s5: INT8 as the next throughput step once the accuracy of  */
/* the attention scores is handled).  The pages fix no format; this one:   */
/* every (token, KV head) row of head_dim values x is stored as head_dim    */
/* int8 codes and one fp32 scale,                                           */
/*   amax = max |x|, inv = 127 / amax, code = rint(x * inv) in [-127, 127],  */
/*   scale = amax / 127                                                     */
/* (fp32 IEEE division and multiply, round half to even; amax 0 gives zero  */
/* codes and scale 0).  A row dequantises to code * scale.  Rows whose amax */
/* is below 127 / FLT_MAX (about 3.7e-37; only bf16 inputs can have them)   */
/* are outside the format.                                                  */
/* Layout: codes k_codes, v_codes int8 [num_blocks][block_size][Hkv][D]     */
/* (the 16-bit caches' layout, one byte per element); scales k_scales,      */
/* v_scales fp32 [num_blocks][Hkv][block_size] (the 16 scales of a 16-token */
/* chunk of one head are one 64-byte run).  All four 16-byte aligned.       */
/*                                                                          */
/* pa_write_kv_int8: for every t with slot = slot_mapping[t] >= 0,           */
/* quantise k[t][h] and v[t][h] (16-bit, [num_tokens][Hkv][D], dtype) into  */
/* row slot of the codes and entry [slot/bs][h][slot%bs] of the scales.     */
/* Same argument rules as pa_write_kv; a slot >= num_blocks*block_size      */
/* writes nothing and sets PA_ERRBIT_INDEX.  Signals its dependents at      */
/* entry (a following pa_decode_int8 may start its set-up early).           */
/* ------------------------------------------------------------------------ */
int pa_write_kv_int8(const void* k, const void* v, const int64_t* slot_mapping, int num_tokens, void* k_codes,
                     void* v_codes, float* k_scales, float* v_scales, int num_blocks, int block_size,
                     int num_kv_heads, int head_dim, int dtype, void* stream);

/* Copy-on-write for the INT8 cache: for each pair i, block pairs[2i+1] of  */
/* the codes and of the scales becomes a bitwise copy of block pairs[2i].   */
int pa_copy_blocks_int8(const int32_t* pairs, int num_pairs, void* k_codes, void* v_codes, float* k_scales,
                        float* v_scales, int num_blocks, int block_size, int num_kv_heads, int head_dim,
                        void* stream);

/* pa_decode_int8: pa_decode over the INT8 cache.  Computes                 */
/*   out[b][h] = sum_t softmax_t(scale * <q[b][h], Kd_b[t]>) Vd_b[t]        */
/* with Kd, Vd the dequantised rows (code * scale) of KV head h/G; q and    */
/* out are 16-bit (dtype), all scores, softmax state and accumulators fp32. */
/* Same work split, workspace rules, argument checks and return codes as    */
/* pa_decode; the workspace size comes from pa_decode_int8_workspace_size   */
/* (or pa_decode_int8_plan).  Internally q is rounded to fp16 after an      */
/* exact power-of-two prescale (its largest magnitude lands in [2^14,       */
/* 2^15)), and the softmax weights enter the V product as fp16 in [0, 1];   */
/* q elements below 2^-28 of the group's largest lose precision.            */
/* ------------------------------------------------------------------------ */
int pa_decode_int8_plan(int batch, int num_q_heads, int num_kv_heads, int head_dim, int max_context_len,
                        int num_partitions_or_0, int* grid_out, int* max_pieces_out, size_t* workspace_bytes_out);
size_t pa_decode_int8_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                     int max_context_len, int num_partitions_or_0);
int pa_decode_int8(const void* q, const void* k_codes, const void* v_codes, const float* k_scales,
                   const float* v_scales, const int32_t* block_tables, int max_blocks_per_seq,
                   const int32_t* context_lens, int batch, int num_q_heads, int num_kv_heads, int head_dim,
                   int block_size, int num_blocks, int max_context_len, float scale, int dtype, void* workspace,
                   size_t workspace_bytes, int num_partitions_or_0, void* out, void* stream);

/* ------------------------------------------------------------------------ */
/* Decode with the context split across devices (P3 s1.1 / s3.1 DCP: each  */
/* device attends over the part of the KV cache it holds; the intermediate */
/* results are gathered from all devices (AllGather) and combined).         */
/* Split rule (the pages give none): logical block j of every sequence      */
/* lives on rank j mod world; on its rank it is local block j / world, so a */
/* rank's blocks form an ordinary paged sequence whose blocks are full but  */
/* the last.  The caller keeps one pool and cache per rank and gathers the  */
/* per-rank results with its collective library (e.g. NCCL all-gather).     */
/*                                                                          */
/* pa_dcp_owner: rank holding token `position` (PA_ERR_INVALID on bad args).*/
/* pa_dcp_local_position: the token's index in its rank's local sequence.  */
/* pa_dcp_local_lens: host int32 arrays; local_lens_out[b] = tokens of      */
/* sequence b (context_lens[b] in all) held by `rank`.                      */
/* ------------------------------------------------------------------------ */
int pa_dcp_owner(int64_t position, int block_size, int world);
int64_t pa_dcp_local_position(int64_t position, int block_size, int world);
int pa_dcp_local_lens(const int32_t* context_lens, int batch, int block_size, int world, int rank,
                      int32_t* local_lens_out);

/* pa_decode_lse: pa_decode that also writes lse_out, fp32 [batch][Hq]       */
/* (device, 4-byte aligned): lse = ln sum_t exp(scale * <q[b][h], K_b[t]>)   */
/* over the sequence's context_lens[b] tokens, -inf when it has none (out   */
/* is then 0).  With a rank's local cache, block tables and local lengths,  */
/* (out, lse) is that rank's intermediate result.  Same rules and return    */
/* codes as pa_decode; lse_out NULL with batch > 0 is PA_ERR_INVALID.       */
int pa_decode_lse(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                  int max_blocks_per_seq, const int32_t* context_lens, int batch, int num_q_heads,
                  int num_kv_heads, int head_dim, int block_size, int num_blocks, int max_context_len, float scale,
                  int dtype, void* workspace, size_t workspace_bytes, int num_partitions_or_0, void* out,
                  float* lse_out, void* stream);

/* pa_merge_attn_states: combine num_parts intermediate results.            */
/* parts: 16-bit (dtype) [num_parts][batch][num_heads][head_dim], lses:     */
/* fp32 [num_parts][batch][num_heads], out: [batch][num_heads][head_dim],   */
/* all device.  out = sum_r exp(lse_r - M) parts_r / sum_r exp(lse_r - M),  */
/* M = max_r lse_r, accumulated in fp32 and rounded to nearest even; a part */
/* with lse -inf adds nothing (its bytes are not read); a row whose parts   */
/* are all -inf is 0.  parts and out 16-byte aligned; out must not overlap  */
/* parts.  One kernel launch on `stream`.                                   */
int pa_merge_attn_states(const void* parts, const float* lses, int num_parts, int batch, int num_heads, int head_dim,
                         int dtype, void* out, void* stream);

/* ------------------------------------------------------------------------ */
/* Chunked prefill (P3 s1.1 / s3.1 PCP: prefill cut into chunks on one       */
/* device).  Sequence b appends C_b = query_start_loc[b+1]-query_start_loc[b]*/
/* query tokens whose K/V were already written (pa_write_kv) so that the    */
/* sequence now holds L_b = context_lens[b] tokens.  Query i of the chunk    */
/* sits at position p = L_b - C_b + i and attends causally to keys 0..p:     */
/*   out[r][h] = sum_{t<=p} softmax_t(scale*<q[r][h], K_b[t][h/G]>) V_b[t][h/G] */
/* with r = query_start_loc[b] + i.                                          */
/* q, out: [total_q_tokens][num_q_heads][head_dim]; query_start_loc: int32   */
/* [batch+1] device, query_start_loc[0] = 0, non-decreasing, last =          */
/* total_q_tokens; C_b <= max_chunk_len and C_b <= L_b.  Requires bf16 or   */
/* f16 with head_dim 128 on the tensor-core path (tcgen05/TMEM).            */
/* Runs as clusters of two CTAs on one TPC (tcgen05.mma cta_group::2), each  */
/* CTA 128 query rows; needs no workspace; asynchronous on `stream`.         */
/* Returns PA_OK (also for batch, total_q_tokens or max_chunk_len = 0),      */
/* PA_ERR_INVALID (negative sizes, null pointers, num_q_heads not a multiple */
/* of num_kv_heads, num_blocks = 0), PA_ERR_UNSUPPORTED (dtype, head_dim !=  */
/* 128, block_size, group size not in {1,2,4,8,16}, caches of 2^31 rows or   */
/* more), PA_ERR_ALIGN (q, caches, out not 16-byte aligned; int32 arrays not */
/* 4-byte aligned) or PA_ERR_CUDA.  On the device, a sequence with L_b above */
/* max_blocks_per_seq*block_size or below C_b, or a block id out of range,   */
/* sets PA_ERRBIT_INDEX (read with pa_device_error); a pipeline wait past    */
/* its 2 s bound sets PA_ERRBIT_TIMEOUT.  Nothing traps.                     */
/* ------------------------------------------------------------------------ */
int pa_prefill_chunk(const void* q, const int32_t* query_start_loc, int total_q_tokens, int max_chunk_len,
                     const void* k_cache, const void* v_cache, const int32_t* block_tables,
                     int max_blocks_per_seq, const int32_t* context_lens, int batch, int num_q_heads,
                     int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale, int dtype,
                     void* out, void* stream);

/* ------------------------------------------------------------------------ */
/* Device error word.  Kernels never trap; a kernel that finds a broken     */
/* device-side invariant (a wait that timed out, an index out of range in   */
/* checked paths) ORs a bit into a per-device error word.  This call        */
/* synchronises the current device, copies the word to *out and clears it. */
/* Bits: 1 = pipeline wait timed out, 2 = index out of range.               */
/* ------------------------------------------------------------------------ */
#define PA_ERRBIT_TIMEOUT 1u
#define PA_ERRBIT_INDEX 2u
int pa_device_error(int* out);

/* ------------------------------------------------------------------------ */
/* Host block pool (P1 s2.1 Block/BlockTable with ref_count; P2 s2.1        */
/* BlockAllocator).  Pure host bookkeeping, no device memory.  Policy: the  */
/* free list starts in `free_order` (NULL = 0..num_blocks-1); allocation    */
/* pops from its head; blocks whose count drops to zero go to its tail.     */
/* A sequence of n tokens holds ceil(n / block_size) blocks.  All calls are */
/* atomic: on error the pool is unchanged.  Not thread-safe.                */
/* ------------------------------------------------------------------------ */
typedef struct pa_pool pa_pool;

typedef struct {
  int64_t num_blocks;
  int64_t free_blocks;
  int64_t used_blocks;    /* blocks with ref_count >= 1 */
  int64_t shared_blocks;  /* blocks with ref_count >= 2 */
  int64_t num_seqs;
  int64_t tokens;         /* sum of sequence lengths */
  int64_t table_refs;     /* sum over sequences of blocks held (== sum of ref counts) */
  int64_t ref_sum;        /* sum of ref counts over all blocks */
  double utilisation;     /* tokens / (table_refs * block_size); 1.0 when empty */
} pa_pool_stats_t;

/* Returns NULL on bad arguments (num_blocks < 0, block_size <= 0, free_order not a permutation). */
pa_pool* pa_pool_create(int num_blocks, int block_size, const int32_t* free_order);
void pa_pool_destroy(pa_pool* pool);

/* New sequence holding num_tokens token slots (ceil(n/bs) blocks, ref_count 1 each). */
int pa_seq_alloc(pa_pool* pool, int64_t seq_id, int num_tokens);

/* New sequence `child` mapping the first ceil(n_prefix/bs) blocks of `parent` (ref_count += 1 each);
   its length is n_prefix (0 <= n_prefix <= parent length). */
int pa_seq_fork(pa_pool* pool, int64_t parent_id, int64_t child_id, int n_prefix);

/* Extend a sequence by n tokens.  slot_mapping_out (host int64 [n], may be NULL) receives the slot of
   each new token.  If the last block is shared and partly filled it is first replaced by a fresh copy
   (copy-on-write): the (src, dst) pair goes to cow_pairs_out (host int32 [2], may be NULL) and
   *num_cow_out (may be NULL) is set to 0 or 1; the caller copies the block (pa_copy_blocks). */
int pa_seq_append(pa_pool* pool, int64_t seq_id, int n, int64_t* slot_mapping_out, int32_t* cow_pairs_out,
                  int* num_cow_out);

/* Extend n sequences in one call: seq_ids[i] by counts[i] tokens, in order i = 0..n-1, with exactly the
   result of n pa_seq_append calls in that order (the per-step append of a decode batch without a call per
   sequence: P2 s3.2 checks the host-side allocation hot path).  All or nothing: an unknown id (PA_ERR_NOT_FOUND), a repeated id or a negative count
   (PA_ERR_INVALID), or a batch needing more blocks than are free (PA_ERR_OOM) leaves the pool unchanged.
   slot_mapping_out (host int64 [sum counts], may be NULL) receives the new tokens' slots in batch order;
   cow_pairs_out (host int32 [n][2], may be NULL) receives the copy-on-write (src, dst) pairs, packed in
   batch order, and *num_cow_out (may be NULL) their number (at most one per sequence). */
int pa_pool_append_batch(pa_pool* pool, const int64_t* seq_ids, const int32_t* counts, int n,
                         int64_t* slot_mapping_out, int32_t* cow_pairs_out, int* num_cow_out);

/* New sequences seq_ids[i] of num_tokens[i] tokens each, as n pa_seq_alloc calls in order would make them.
   All or nothing: a live or repeated id (PA_ERR_NOT_FOUND / PA_ERR_INVALID), a negative count
   (PA_ERR_INVALID) or too few free blocks for the whole batch (PA_ERR_OOM) leaves the pool unchanged. */
int pa_pool_alloc_batch(pa_pool* pool, const int64_t* seq_ids, const int32_t* num_tokens, int n);

/* Drop sequences seq_ids[0..n), as n pa_seq_free calls in order would.  All or nothing: an unknown
   (PA_ERR_NOT_FOUND) or repeated (PA_ERR_INVALID) id leaves the pool unchanged. */
int pa_pool_free_batch(pa_pool* pool, const int64_t* seq_ids, int n);

/* Drop a sequence: ref_count -= 1 on each of its blocks; blocks reaching 0 return to the free list. */
int pa_seq_free(pa_pool* pool, int64_t seq_id);

/* Length of a sequence (tokens) in *len_out and blocks held in *blocks_out (either may be NULL). */
int pa_seq_info(const pa_pool* pool, int64_t seq_id, int* len_out, int* blocks_out);

/* Export block table rows for seq_ids[0..n): out is host int32 [n][max_blocks], padded with -1;
   ctx_lens_out (host int32 [n], may be NULL) receives the lengths.  PA_ERR_INVALID if a row is too short. */
int pa_pool_block_table(const pa_pool* pool, const int64_t* seq_ids, int n, int32_t* out, int max_blocks,
                        int32_t* ctx_lens_out);

/* Reference count of one physical block (or -1 for an id out of range). */
int pa_pool_ref_count(const pa_pool* pool, int block_id);

int pa_pool_stats(const pa_pool* pool, pa_pool_stats_t* out);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_ATTN_H */
