/*
 * Exact attention forward (bf16 and FP8, on device or host buffers), backward, paged-KV
 * decoding and the partial-result merge of ring attention for NVIDIA B200 (sm_100a): C ABI.
 *
 * Computes, for every batch b, query head h and query row i,
 *
 *     out[b,h,i,:] = sum_j softmax_j(scale * q[b,h,i,:] . k[b,g(h),j,:] + mask(i,j)) * v[b,g(h),j,:]
 *     lse[b,h,i]   = ln sum_{j visible} exp(scale * q[b,h,i,:] . k[b,g(h),j,:])
 *
 * which is the masked softmax attention of "Efficient attention: long context and
 * sub-quadratic variants" (stanleyjacob.dev), section "Implementation, twice"
 * (masked_attention: masked scores are -inf before the softmax, each row is
 * renormalised over its visible keys), computed tile by tile with an online
 * softmax so the N x N score matrix never reaches HBM (same page, section
 * "FlashAttention: exact attention, IO-aware").
 *
 * Masks (mask(i,j) = 0 where visible, -inf elsewhere):
 *   ATTN_MASK_FULL            every key;
 *   ATTN_MASK_CAUSAL          j <= i ("Efficient Attention: Flash Attention, Sliding
 *                             Window, Sparse", creativeworksofknowledge.com, section "Code":
 *                             is_causal=True);
 *   ATTN_MASK_SLIDING_WINDOW  i - window < j <= i (stanleyjacob.dev, section
 *                             "Sliding-window and local attention" and sliding_window_mask);
 *                             a window >= N is exactly causal and is run as causal.
 * Head sharing (GQA/MQA): query head h reads key/value head g(h) = h / (Hq / Hkv)
 * ("Attention Mechanism Variants Beyond Self-Attention", tempatgunting.com, section
 * "Multi-Query and Grouped-Query Attention": repeat_interleave on the head axis).
 * The log-sum-exp output is not on those pages; it is the natural-log normaliser of
 * each row's softmax, written so a caller can merge or recompute partial results.
 */
#ifndef ATTN_B200_ATTN_H_
#define ATTN_B200_ATTN_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_MASK_FULL = 0,
  ATTN_MASK_CAUSAL = 1,
  ATTN_MASK_SLIDING_WINDOW = 2
} attn_mask_kind;

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad mask, window < 1, scale not finite or <= 0,
                                overlapping buffers */
  ATTN_ERR_UNSUPPORTED = 2,  /* head dimension other than 64 or 128, or no sm_100 device */
  ATTN_ERR_MISALIGNED = 3,   /* q, k, v or out not 16-byte aligned, lse not 4-byte aligned */
  ATTN_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed (launch, tensor-map encode) */
  ATTN_ERR_TIMEOUT = 5,      /* a device-side wait gave up (reported by attn_debug_error) */
  ATTN_ERR_RANGE = 6         /* a V value that fp16 cannot hold (magnitude >= 2^16, or not finite) met
                                the default fp16 P V product (reported by attn_debug_error) */
} attn_status;

/*
 * attn_fwd: enqueue the forward on `stream` and return immediately.
 *
 *   q    device pointer, bf16, [B, Hq,  N, d], contiguous (d fastest), 16-byte aligned
 *   k    device pointer, bf16, [B, Hkv, N, d], contiguous, 16-byte aligned
 *   v    device pointer, bf16, [B, Hkv, N, d], contiguous, 16-byte aligned
 *   out  device pointer, bf16, [B, Hq,  N, d], contiguous, 16-byte aligned; fully overwritten
 *   lse  device pointer, fp32, [B, Hq,  N],    contiguous, 4-byte aligned; fully overwritten
 *   B, Hq, Hkv, N >= 1; Hq % Hkv == 0; d in {64, 128}
 *   scale      finite and > 0 (usually 1/sqrt(d)); multiplies q.k before the mask
 *   mask_kind  an attn_mask_kind
 *   window     >= 1 when mask_kind == ATTN_MASK_SLIDING_WINDOW, ignored otherwise
 *   stream     CUDA stream (0 = legacy default stream) of the current device, which
 *              must own all five buffers
 *
 * Ownership: the caller owns every buffer. The library allocates no device memory and
 * never synchronises; out and lse are written by the kernel when the stream reaches it.
 * out and lse must not overlap each other or the inputs (ATTN_ERR_INVALID_ARG).
 * Precision: scores and sums are fp32; the softmax weights P go to the tensor core as
 * fp16 (11 significant bits), with V converted to fp16 on chip, and out is rounded once
 * to bf16. V values must therefore have magnitude below 2^16 (every finite bf16 value
 * up to 65280 qualifies); a larger or non-finite V value makes the launch's result
 * undefined and is reported by attn_debug_error as ATTN_ERR_RANGE. attn_fwd_ex with
 * p_bf16 = 1 takes any V, with P rounded to bf16 instead (8 significant bits: out can
 * then be off by about one bf16 ulp of a value near 1 where one or two keys dominate).
 * Errors: every argument is checked before anything is enqueued; on error nothing is
 * launched and the status says why. ATTN_ERR_CUDA reports a failed launch. Device-side
 * waits are bounded (about 2 s); a wait that gives up makes the kernel stop early and
 * leave a code that attn_debug_error returns as ATTN_ERR_TIMEOUT.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
             int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d,
             float scale, int mask_kind, int64_t window, cudaStream_t stream);

/* Options for attn_fwd_ex (and the _ex forms of the other calls, which say which
   fields they read). Zero-initialise, then set what is needed. */
typedef struct {
  uint64_t wait_timeout_ns; /* bound of every device-side wait; 0 = default (2 s) */
  int inject_stall;         /* test hook: 1 = the loader issues no copies, so every consumer
                               wait runs out and the kernel exits with ATTN_ERR_TIMEOUT
                               pending in attn_debug_error; nothing faults or hangs */
  int grid_ctas;            /* number of persistent CTAs; 0 = one per SM */
  unsigned int* item_visits; /* test hook (forward): NULL, or a device array of
                               attn_fwd_num_work_items() counters, each incremented once
                               per visit of its work item (the caller zeroes it) */
  int p_bf16;               /* 1 = P and V go to the P V product as bf16 (any V value, coarser
                               P); 0 = fp16 (default; |V| below 2^16). bf16 inputs only */
  int out_fp32;             /* forward: 1 = out is fp32 [B, Hq, N, d] (16-byte aligned) and
                               receives O / l unrounded, for partial results that are merged
                               afterwards (attn_merge mode 2 or 3); 0 = bf16 out */
  int64_t key_offset;       /* forward, causal and window masks: query row i sits at key
                               position i + key_offset (>= 0), so it sees keys j <= i + key_offset
                               (and, with a window, j > i + key_offset - window), e.g. a query
                               block against an earlier key block in ring attention; rows that
                               see no key end with out 0 and lse -inf. 0 = the square masks */
  int bwd_deterministic;    /* backward, d = 128: 1 = the two-kernel path (query-tile dQ kernel,
                               key-tile dK/dV kernel; seven matmuls per pair, dq bitwise
                               reproducible, workspace 4 B Hq N bytes, 4-byte aligned);
                               0 = the fused key-tile kernel where Hq == Hkv (default) */
} attn_fwd_options;

/* attn_fwd with options (same arguments, same checks); opts may be NULL. */
int attn_fwd_ex(const void* q, const void* k, const void* v, void* out, float* lse,
                int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d,
                float scale, int mask_kind, int64_t window, cudaStream_t stream,
                const attn_fwd_options* opts);

/*
 * attn_fwd_fp8: the same forward with E4M3 inputs. q, k, v hold 8-bit E4M3 codes (OCP
 * format: bias 7, no infinities, largest magnitude 448) in the layouts of attn_fwd, with
 * one scale per tensor: element value = E4M3(code) * q_scale (k_scale, v_scale). The
 * result is the exact attention of those values (scale multiplies their q.k), out bf16
 * and lse fp32 as attn_fwd. The pages name FP8 inputs as a feature of the production
 * kernel line ("Efficient Attention: Flash Attention, Sliding Window, Sparse",
 * creativeworksofknowledge.com, section "Flash Attention (exact, memory-efficient)").
 * Inside, q.k runs on E4M3 tensor-core products and P is rounded to E4M3 (times 2^8)
 * for the product with V; accumulation is fp32.
 *
 *   q, k, v      device pointers to uint8 codes, [B, Hq|Hkv, N, d], contiguous, 16-byte aligned
 *   q_scale, k_scale, v_scale   finite and > 0
 *   d            128 only (ATTN_ERR_UNSUPPORTED otherwise)
 *   everything else as attn_fwd
 */
int attn_fwd_fp8(const void* q, const void* k, const void* v, float q_scale, float k_scale, float v_scale,
                 void* out, float* lse, int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d,
                 float scale, int mask_kind, int64_t window, cudaStream_t stream);
/* attn_fwd_fp8 with options (as attn_fwd_ex); opts may be NULL. */
int attn_fwd_fp8_ex(const void* q, const void* k, const void* v, float q_scale, float k_scale, float v_scale,
                    void* out, float* lse, int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d,
                    float scale, int mask_kind, int64_t window, cudaStream_t stream,
                    const attn_fwd_options* opts);

/*
 * attn_fwd_host: attn_fwd on HOST buffers, with the copies overlapped with the work.
 * The (batch, key/value head) units are independent and a contiguous range of units is a
 * contiguous range of every tensor, so the job is cut into `chunks` ranges. Each range is
 * uploaded on a copy stream. Its forward runs on `stream` once it has arrived, and its out
 * and lse go back on a second copy stream once computed. Different chunks' uploads, kernels
 * and downloads therefore run at the same time.
 *
 *   hq, hk, hv    host pointers, layouts and types of attn_fwd's q, k, v (page-locked
 *                 memory lets the copies overlap; pageable memory works, more slowly)
 *   hout, hlse    host pointers, layouts of attn_fwd's out and lse; must not overlap the
 *                 host inputs or each other
 *   dq, dk, dv, dout, dlse   device staging buffers with attn_fwd's sizes, alignment and
 *                 overlap rules (owned by the caller; their contents are overwritten);
 *                 since the uploads write dq, dk and dv, these three must not overlap
 *                 one another either (ATTN_ERR_INVALID_ARG)
 *   B ... window  as attn_fwd
 *   chunks        number of ranges, >= 0; 0 = 8; more than B * Hkv means B * Hkv
 *   stream        CUDA stream of the current device
 *
 * Everything is enqueued and the call returns. hout and hlse are complete when `stream`
 * reaches the point after the call: `stream` waits for the last download. The call does
 * not block the host unless the host memory is pageable, in which case the runtime may
 * copy synchronously. The library keeps two copy streams per device, created on first
 * use, and allocates no memory. Errors: arguments are checked before anything is
 * enqueued, as in attn_fwd, and so is the device (ATTN_ERR_UNSUPPORTED unless sm_100).
 * If something fails part way, its status is returned: ATTN_ERR_CUDA for a copy, the
 * chunk's attn_fwd status for a launch. `stream` is still ordered after whatever had been
 * enqueued.
 */
int attn_fwd_host(const void* hq, const void* hk, const void* hv, void* hout, float* hlse,
                  void* dq, void* dk, void* dv, void* dout, float* dlse,
                  int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d,
                  float scale, int mask_kind, int64_t window, int64_t chunks, cudaStream_t stream);
/* attn_fwd_host for the E4M3 inputs of attn_fwd_fp8 (same scales, same restrictions). */
int attn_fwd_fp8_host(const void* hq, const void* hk, const void* hv,
                      float q_scale, float k_scale, float v_scale, void* hout, float* hlse,
                      void* dq, void* dk, void* dv, void* dout, float* dlse,
                      int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d,
                      float scale, int mask_kind, int64_t window, int64_t chunks, cudaStream_t stream);

/*
 * attn_merge: fold one partial attention result into an accumulator, the combining step of
 * ring attention ("Attention Mechanism Variants Beyond Self-Attention", tempatgunting.com,
 * section "Ring Attention for Very Long Sequences": each GPU holds a chunk of the sequence
 * and key/value blocks rotate around a ring). For each row, with partial (O_p, lse_p) over
 * one set of keys and accumulated (O_a, lse_a) over a disjoint set,
 *   lse = ln(e^lse_a + e^lse_p),  O = e^(lse_a - lse) O_a + e^(lse_p - lse) O_p,
 * the attention over the union (each partial O is normalised by its own softmax sum).
 *
 *   acc_out   device, fp32 [rows, d], 16-byte aligned; read (mode 1) and written
 *   acc_lse   device, fp32 [rows], natural log; read (mode 1) and written
 *   part_out  device, [rows, d] (attn_fwd's out for one block of keys): bf16, 8-byte aligned
 *             (modes 0, 1), or fp32, 16-byte aligned (modes 2, 3: attn_fwd_ex with out_fp32)
 *   part_lse  device, fp32 [rows] (attn_fwd's lse for the same block)
 *   out       device, bf16 [rows, d], 8-byte aligned, or NULL: when given, the merged rows are
 *             also written here rounded to bf16 (it may be part_out itself)
 *   rows      1 .. 2^33; d in {64, 128}
 *   mode      0: the accumulator is set to the partial; 1: the partial is merged into it;
 *             2, 3: the same with an fp32 partial (no bf16 rounding before the merge)
 * Errors as attn_fwd; nothing is allocated and nothing synchronises.
 */
int attn_merge(float* acc_out, float* acc_lse, const void* part_out, const float* part_lse, void* out,
               int64_t rows, int64_t d, int mode, cudaStream_t stream);
/* Human-readable name of an attn_status value (static string, never NULL). */
const char* attn_status_string(int status);

/*
 * attn_debug_error: synchronise `stream`, read and clear the device error word of the
 * current device. Returns ATTN_OK if no device wait gave up since the last call,
 * ATTN_ERR_TIMEOUT if one did (the raw code, which names the waiting role, goes to
 * *device_code when device_code is not NULL), ATTN_ERR_RANGE if a V value beyond the
 * fp16 range met the fp16 P V product, ATTN_ERR_CUDA if the synchronisation itself
 * failed. The error word is one per device, shared by every stream and every forward
 * launch on it (attn_fwd, attn_fwd_fp8, the host-buffer calls): it keeps the first code
 * any of them records until a call of this function clears it, and this function waits
 * only for `stream`. With launches on several streams, synchronise them all before
 * reading it, or a code may be seen (and cleared) by the call for another stream.
 */
int attn_debug_error(cudaStream_t stream, int* device_code);

/* Number of persistent work items a launch with these sizes schedules (host-only
   helper for tests and tools; returns -1 on invalid sizes). */
int64_t attn_fwd_num_work_items(int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d,
                                int mask_kind, int64_t window);

/*
 * attn_bwd: enqueue the backward pass on `stream`: the gradients of sum(dout * out)
 * with respect to q, k and v for the forward above (same masks, head map and scale).
 * With S = scale q k^T (masked entries -inf) and P = exp(S - lse) per query row, the
 * chain rule gives dV = P^T dO, dP = dO V^T, dS = P (dP - D) with D_i = dO_i . O_i,
 * dQ = scale dS K and dK = scale dS^T Q; a KV head's dK, dV sum over the query heads
 * that read it. The pages name a recompute-based backward pass as part of the
 * production kernel line ("Efficient attention: long context and sub-quadratic
 * variants", stanleyjacob.dev, section "Against the real libraries"); P is recomputed
 * from lse, never stored.
 *
 *   q, k, v    as attn_fwd (bf16, contiguous, 16-byte aligned)
 *   out, lse   attn_fwd's outputs for these q, k, v, scale and mask (read only)
 *   dout       device pointer, bf16, [B, Hq, N, d], contiguous, 16-byte aligned
 *   dq         device pointer, bf16, [B, Hq,  N, d], 16-byte aligned; fully overwritten
 *   dk, dv     device pointers, bf16, [B, Hkv, N, d], 16-byte aligned; fully overwritten
 *   workspace  device pointer owned by the caller; attn_bwd_workspace_bytes(B, Hq, N) bytes,
 *              16-byte aligned, always suffice. The minimum: on the two-kernel path (d = 64,
 *              Hq != Hkv, or bwd_deterministic) 4 B Hq N bytes, 4-byte aligned, holding D
 *              (fp32 [B, Hq, N]); on the fused path the full size, 16-byte aligned: D, then (from
 *              the next 256-byte boundary) an fp32 [B, Hq, N, 128] dQ accumulator that the
 *              call zeroes and fills. Not to be reused until the stream has passed the call.
 *   B, Hq, Hkv, N, d, scale, mask_kind, window, stream: as attn_fwd
 *
 * Launches: D, then for d = 128 with Hq == Hkv a fused kernel that forms P and dS once
 * per (query, key) pair (one CTA per 128-key tile: dK, dV in TMEM; dQ's partial sums of
 * each tile added into the accumulator with fp32 global reductions) and a kernel rounding
 * dQ to bf16; otherwise (d = 64, grouped heads) a query-tile kernel for dQ and a key-tile
 * kernel for dK, dV. On the fused path the order of the fp32 additions into dQ varies
 * from run to run, so dq is reproducible only up to the rounding of those sums (dk and dv
 * are bitwise reproducible); attn_bwd_ex with bwd_deterministic = 1 takes the two-kernel
 * path there too.
 *
 * The library allocates nothing. Outputs and the workspace must not overlap each other
 * or the inputs (ATTN_ERR_INVALID_ARG). Errors and bounded waits as attn_fwd; a wait
 * that gives up leaves a code that attn_bwd_debug_error returns as ATTN_ERR_TIMEOUT.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
             const void* dout, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
             int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d,
             float scale, int mask_kind, int64_t window, cudaStream_t stream);

/* attn_bwd with options (wait bound and CTA count as for attn_fwd_ex, and
   bwd_deterministic; the other fields are ignored); opts may be NULL. */
int attn_bwd_ex(const void* q, const void* k, const void* v, const void* out, const float* lse,
                const void* dout, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d,
                float scale, int mask_kind, int64_t window, cudaStream_t stream,
                const attn_fwd_options* opts);

/* Workspace bytes attn_bwd needs for any supported d: 4 B Hq N rounded up to 256, plus
   4 B Hq N 128 (the d = 128 dQ accumulator); 0 for invalid sizes or a total beyond 2^61. */
size_t attn_bwd_workspace_bytes(int64_t B, int64_t Hq, int64_t N);

/* attn_debug_error for the backward kernels' error word (same contract). */
int attn_bwd_debug_error(cudaStream_t stream, int* device_code);
/*
 * attn_decode: enqueue one decoding step on `stream`: the Nq new tokens of each of B
 * sequences attend to that sequence's cached keys and values, which are stored in
 * fixed-size pages reached through a per-sequence page table ("Efficient attention:
 * long context and sub-quadratic variants", stanleyjacob.dev, section "FlashAttention:
 * exact attention, IO-aware", PagedAttention paragraph; "Efficient Attention",
 * giftedprocrastinator.com, section "What it does": the KV cache keeps past keys and
 * values so a new token does not recompute them). Nothing is approximated: the result is
 * the masked softmax attention of attn_fwd for the new tokens' rows.
 *
 * With L_b = seq_lens[b] cached positions (the new tokens included), new token t of
 * sequence b is at position L_b - Nq + t and sees cached positions j with
 *   ATTN_MASK_FULL            0 <= j < L_b;
 *   ATTN_MASK_CAUSAL          j <= L_b - Nq + t;
 *   ATTN_MASK_SLIDING_WINDOW  L_b - Nq + t - window < j <= L_b - Nq + t.
 * Position j of sequence b lives in physical page block_table[b][j / page_size], slot
 * j % page_size. Only pages holding positions from lo_b = max(0, L_b - Nq - window + 1)
 * (0 without a window) to L_b - 1 are looked up or read: under a sliding window a caller
 * may recycle older pages and leave their table entries stale (a rolling window buffer);
 * slots past L_b in the last page may hold anything.
 *
 *   q            device, bf16, [B, Hq, Nq, d], contiguous, 16-byte aligned
 *   k_cache      device, bf16, [num_pages, Hkv, page_size, d], contiguous, 16-byte aligned
 *   v_cache      device, bf16, same shape as k_cache
 *   block_table  device, int32, [B, max_pages_per_seq], 4-byte aligned
 *   seq_lens     device, int32, [B], 4-byte aligned; Nq <= seq_lens[b] <= max_pages_per_seq *
 *                page_size (violations are reported by attn_decode_debug_error as
 *                ATTN_ERR_INVALID_ARG and leave those rows zero with lse = -inf)
 *   out          device, bf16, [B, Hq, Nq, d], 16-byte aligned; fully overwritten
 *   lse          device, fp32, [B, Hq, Nq], 4-byte aligned; natural-log normaliser of each row
 *   workspace    device, 16-byte aligned, at least attn_decode_workspace_bytes(B, Hq, Nq, d,
 *                num_splits) bytes, owned by the caller. Its first 256 bytes hold the counter
 *                that hands work items to the SMs: they must be zero before the first call that
 *                uses the workspace, and every call leaves them zero again. The rest holds the
 *                splits' partial results until the merge launch of the same call has read them.
 *                Calls that share a workspace must not run concurrently.
 *   Hq % Hkv == 0; query head h reads KV head h / (Hq / Hkv); d in {64, 128};
 *   page_size in {16, 32, 64, 128, 256}
 *   num_splits   1..4096: each sequence's visible key range is cut into this many parts
 *                processed in parallel and merged by their log-sum-exp
 *                (attn_decode_num_splits suggests one)
 *   scale, mask_kind, window, stream: as attn_fwd
 *
 * Ownership: the caller owns every buffer; the library allocates nothing and never
 * synchronises. Outputs and the workspace must not overlap each other or the inputs
 * (ATTN_ERR_INVALID_ARG). A page-table entry outside [0, num_pages) that the step needs
 * is reported by attn_decode_debug_error as ATTN_ERR_INVALID_ARG (the step's result is
 * then undefined, but nothing outside the given buffers is read). Precision: scores, sums
 * and the split partials are fp32; P goes to the P V product rounded to bf16 (RNE), so,
 * unlike attn_fwd, a row dominated by a few keys can be off by about one bf16 ulp of out
 * (the step is bound by HBM reads, and an fp16 copy of V in shared memory would hold each
 * V slot of the load ring longer, costing 15-40 % of the bandwidth). Any bf16 V is taken.
 * Errors, bounded waits and ATTN_ERR_TIMEOUT as attn_fwd.
 */
int attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                const int32_t* seq_lens, void* out, float* lse, void* workspace, size_t workspace_bytes,
                int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t d,
                int64_t num_pages, int64_t page_size, int64_t max_pages_per_seq, int64_t num_splits,
                float scale, int mask_kind, int64_t window, cudaStream_t stream);
/* attn_decode with options (wait bound and CTA count as for attn_fwd_ex; the other
   fields are ignored); opts may be NULL. */
int attn_decode_ex(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                   const int32_t* seq_lens, void* out, float* lse, void* workspace, size_t workspace_bytes,
                   int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t d,
                   int64_t num_pages, int64_t page_size, int64_t max_pages_per_seq, int64_t num_splits,
                   float scale, int mask_kind, int64_t window, cudaStream_t stream,
                   const attn_fwd_options* opts);
/* Workspace bytes attn_decode needs for num_splits (256 + the partial results when
   num_splits > 1; 0 on invalid sizes). */
size_t attn_decode_workspace_bytes(int64_t B, int64_t Hq, int64_t Nq, int64_t d, int64_t num_splits);
/* Suggested num_splits for a step whose longest sequence has max_seq_len cached positions,
   on the current device: one wave of work items when B * Hkv (times the query-row chunks)
   is below the SM count, otherwise splits of at most 64 128-key tiles; never a split
   shorter than four tiles; -1 on invalid sizes. Host-only. */
int64_t attn_decode_num_splits(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t max_seq_len,
                               int mask_kind, int64_t window);
/* attn_debug_error for the decoding kernel's error word (one per device, shared like the
   forward's): ATTN_ERR_TIMEOUT for a wait that gave up, ATTN_ERR_INVALID_ARG for a bad
   sequence length or page-table entry. */
int attn_decode_debug_error(cudaStream_t stream, int* device_code);

/*
 * attn_decode_static: attn_decode without a caller workspace, for callers that cannot
 * allocate device memory. (The pages have no counterpart: this is a deployment variant
 * of the decoding step above, with the same result.)
 *
 * Who needs it: code that runs inside a host program which owns all device memory and
 * hands the code only its input and output buffers -- an inference-server plugin, an
 * embedded runtime with a fixed memory plan, a language binding without a device
 * allocator. There a cudaMalloc is either not permitted, breaks the owner's memory plan,
 * or synchronises the device at a moment the caller does not control.
 *
 * Instead of `workspace`, the call uses a scratch array that the library itself defines
 * in device memory: ATTN_DECODE_STATIC_SCRATCH_BYTES bytes, held by every GPU that loads
 * the library until the process exits. Nothing is allocated by the call: no cudaMalloc,
 * no cudaFree, no allocating library routine.
 *
 *   arguments    those of attn_decode without workspace and workspace_bytes, with the
 *                same meaning, layouts, checks and errors
 *   size limit   attn_decode_workspace_bytes(B, Hq, Nq, d, num_splits) must not exceed
 *                ATTN_DECODE_STATIC_SCRATCH_BYTES; a larger step is refused with
 *                ATTN_ERR_UNSUPPORTED before anything is enqueued (use fewer splits, a
 *                smaller batch, or attn_decode with a workspace)
 *
 * Set-up: the first call on a device, with that device current, looks up the device
 * address of the array (once per device); make that first call before any stream capture.
 * Every call then enqueues, on `stream`, a clear of the array's work counter followed by
 * the decoding launches. If attn_decode's argument checks then refuse the call, that
 * clear, which touches only the library's own array, may already be enqueued.
 * Every call on a device shares the one array, and the array keeps the last call's
 * partial results: calls that overlap on the GPU (other streams, other host threads)
 * race on it and give wrong results. Order them, e.g. on one stream.
 */
#define ATTN_DECODE_STATIC_SCRATCH_BYTES (8u * 1024u * 1024u)
int attn_decode_static(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                       const int32_t* seq_lens, void* out, float* lse,
                       int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t d,
                       int64_t num_pages, int64_t page_size, int64_t max_pages_per_seq, int64_t num_splits,
                       float scale, int mask_kind, int64_t window, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_ATTN_H_ */
