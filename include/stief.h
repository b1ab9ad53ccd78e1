/*
 * stief.h -- C ABI of the B200 (sm_100a) StiefAttention latent-KV decode library.
 *
 * The operation comes from "Don't be so Stief! Learning KV Cache low-rank
 * approximation over the Stiefel manifold" (StiefAttention technical summary,
 * "Mecanismo Central" / "Kernmechanismus"):
 *   item 2 -- the projection bases P_K (d x r_K) and P_V (d x r_V) have
 *             orthonormal columns (points on the Stiefel manifold);
 *   item 5 -- keys and values are stored compressed, K_down = K . P_K and
 *             V_down = V . P_V, and the full dimensions are reconstructed on the
 *             fly, K~ = K_down . P_K^T, V~ = V_down . P_V^T, before attention.
 * The pages give no interface, precision, scale, head mapping or layout.  This
 * library fixes them as follows:
 *   - one basis pair per KV head, bf16, row-major [Hkv][d][r];
 *   - scores are scaled by 1/sqrt(d), d the full head dimension;
 *   - grouped-query attention with contiguous groups: query head h reads KV
 *     head h / (Hq / Hkv);
 *   - the latent cache is bf16, row-major [B][Hkv][L_max][r] (one row per
 *     token); all arithmetic accumulates in fp32; outputs are bf16 (RNE).
 *
 * Conventions for every call:
 *   - "bf16" arguments are arrays of IEEE bfloat16 bit patterns (uint16_t).
 *   - Every pointer is caller-owned DEVICE memory on the current CUDA device,
 *     dense (no strides), and 16-byte aligned.  The library never allocates,
 *     frees or retains memory and keeps no state between calls.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream).
 *     A call that returns an error from argument checking launches nothing.
 *   - Supported: d == 128; 16 <= r_K, r_V <= 128 with r % 16 == 0; Hq % Hkv == 0;
 *     1 <= Hq / Hkv <= 64; B, Hkv >= 1; for the decode calls B <= 65535 and
 *     B * Hkv * L_max < 2^31 (cache rows are addressed with 32-bit copy coordinates).
 *   - `dev_status` (may be NULL) is a device uint32 word.  Kernels OR the
 *     STIEF_DEV_* bits below into it when they meet a condition that host-side
 *     checks cannot see.  The library never clears it: the caller zeroes it
 *     and reads it back with stief_read_device_status().
 *   - Calls on one stream are ordered; concurrent calls on different streams
 *     must not share output or workspace buffers.
 */
#ifndef STIEF_H
#define STIEF_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define STIEF_API __attribute__((visibility("default")))
#else
#define STIEF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* The same type as cudaStream_t (a pointer to the runtime's opaque stream). */
typedef struct CUstream_st* stief_stream_t;

typedef enum stief_status {
    STIEF_OK = 0,
    STIEF_ERR_INVALID_ARG = 1,      /* null pointer, bad size or unsupported shape */
    STIEF_ERR_ALIGNMENT = 2,        /* a pointer is not 16-byte aligned */
    STIEF_ERR_CAPACITY = 3,         /* max_seq_len > L_max, or T > L_max */
    STIEF_ERR_WORKSPACE = 4,        /* workspace missing or smaller than required */
    STIEF_ERR_CUDA = 5,             /* a CUDA runtime call failed (launch, attribute) */
    STIEF_ERR_DEVICE_STATUS = 6,    /* stief_read_device_status found a non-zero word */
    STIEF_ERR_UNSUPPORTED_DEVICE = 7 /* current device is not compute capability 10.0 */
} stief_status;

/* Bits kernels OR into *dev_status. */
#define STIEF_DEV_CAPACITY_OVERFLOW 0x1u /* compress: seq_lens[b] + T > L_max; that
                                            sequence was left untouched */
#define STIEF_DEV_WAIT_TIMEOUT 0x2u      /* a bounded wait on an asynchronous copy or
                                            tensor-core completion gave up; the call's
                                            results are undefined (a compress may still
                                            have advanced the lengths: put them back and
                                            call again; a decode: zero the workspace) */
#define STIEF_DEV_BAD_LENGTH 0x4u        /* a seq_lens entry was negative or > L_max
                                            (decode: that sequence's output is zero;
                                            compress: it is left untouched) */
#define STIEF_DEV_SMEM_ALIGN 0x8u        /* decode: dynamic shared memory was not 1 KiB
                                            aligned as the swizzled key tiles need;
                                            nothing was computed */

/*
 * stief_compress_append -- compressed storage of new keys and values
 * (StiefAttention technical summary, "Mecanismo Central" item 5: K_down = K P_K).
 *
 * For every sequence b and KV head h, projects the T new rows
 *     k_lat[b][h][seq_lens[b] + t][:] = bf16_RNE( k_new[b][h][t][:] . P_K[h] )
 *     v_lat[b][h][seq_lens[b] + t][:] = bf16_RNE( v_new[b][h][t][:] . P_V[h] )
 * for t < T (fp32 accumulation), then sets seq_lens[b] += T.  Rows outside
 * [seq_lens[b], seq_lens[b] + T) are not touched.
 *
 *   k_new, v_new : bf16 [B][Hkv][T][d]              (read)
 *   P_K, P_V     : bf16 [Hkv][d][rK], [Hkv][d][rV]  (read)
 *   k_lat, v_lat : bf16 [B][Hkv][L_max][rK], [B][Hkv][L_max][rV]  (written)
 *   seq_lens     : int32 [B] on the device          (read, then advanced by T)
 *   T            : rows per (sequence, head); T == 0 is a no-op returning OK
 *
 * A sequence whose seq_lens[b] + T exceeds L_max (or whose length is negative)
 * is skipped entirely -- no row written, length unchanged -- and
 * STIEF_DEV_CAPACITY_OVERFLOW (or STIEF_DEV_BAD_LENGTH) is set in *dev_status.
 * Small T runs on CUDA cores; prefill-sized T (>= 128) runs as a tcgen05
 * tensor-core GEMM with the accumulator in tensor memory.  That kernel is
 * launched as a programmatic dependent of the preceding work in the stream and
 * stages P_K and P_V before waiting for it: the bases must not be written by the
 * kernel that immediately precedes the call if that kernel lets its dependents
 * start early (this library's kernels never write the bases).  The call ends with
 * a small kernel that advances the lengths once every projection CTA has read
 * them; it lets the next kernel in the stream start early (that kernel's inputs
 * are read after its own dependency wait).  The library notes per stream that its
 * last launch there was a compress, and the decode call that follows requests no
 * cache row before its wait.
 * Returns STIEF_OK or an argument error (nothing launched).
 */
STIEF_API stief_status stief_compress_append(const uint16_t* k_new, const uint16_t* v_new,
                                   const uint16_t* P_K, const uint16_t* P_V,
                                   uint16_t* k_lat, uint16_t* v_lat, int32_t* seq_lens,
                                   int B, int Hkv, int T, int d, int rK, int rV, int L_max,
                                   uint32_t* dev_status, stief_stream_t stream);

/*
 * stief_decode_max_splits -- the largest split count a decode over sequences of
 * at most max_seq_len tokens may use (explicit or automatic).  Pure host
 * function.  Returns 0 for invalid arguments.
 */
STIEF_API int stief_decode_max_splits(int max_seq_len);

/*
 * stief_decode_auto_splits -- the split count stief_decode_attention picks when
 * num_splits == 0, for a device with num_sms streaming multiprocessors.  Pure
 * host function (no CUDA call).  Returns 0 for invalid arguments.
 */
STIEF_API int stief_decode_auto_splits(int B, int Hq, int Hkv, int max_seq_len, int num_sms);

/*
 * stief_decode_workspace_bytes -- bytes of device workspace stief_decode_attention
 * needs for these sizes, for any split count it may use (at most
 * stief_decode_max_splits(max_seq_len)).  The workspace holds one ticket counter
 * per (sequence, KV head, query sub-group) and one per sequence (padded together to
 * 256 bytes), followed by the per-split partial states: for each query head, the
 * split's latent output o~ scaled to its running maximum (r_V values), that maximum
 * and its sum.  When the whole grid fits on the GPU at once they are 8-byte words
 * (an fp32 value and a tag saying it was written; the CTA of split s merges heads
 * s, s + S, ... as soon as every split's words are there, then zeroes them); otherwise
 * r_V + 4 floats, merged by the last CTA to take a ticket.  Either way the size is
 * B*Hkv*ceil(G/G_T)*G_T*splits*(d+2)*8 bytes after the counters (G = Hq/Hkv, G_T the
 * smallest of 1, 2, 4, 8 that is >= min(G, 8), splits = stief_decode_max_splits), so
 * rV is validated but does not change it.  The same workspace serves
 * stief_append_decode and stief_decode_latent.  Pure host function.  Returns 0 for
 * invalid arguments.
 */
STIEF_API size_t stief_decode_workspace_bytes(int B, int Hq, int Hkv, int rV, int max_seq_len);

/*
 * stief_decode_attention -- one autoregressive decode step over the latent cache
 * (StiefAttention technical summary, "Mecanismo Central" item 5: attention over
 * K~ = K_down P_K^T and V~ = V_down P_V^T).
 *
 * For every sequence b and query head h (KV head g = h / (Hq/Hkv), L = seq_lens[b]):
 *     s_t = q[b][h] . K~_t / sqrt(d)                       t < L
 *     out[b][h] = bf16_RNE( sum_t softmax(s)_t V~_t )
 * computed without materialising K~ or V~:
 *     q~ = q[b][h] . P_K[g]                  (per CTA)
 *     s_t = q~ . K_down[b][g][t] / sqrt(d)
 *     o~ = sum_t softmax(s)_t V_down[b][g][t] (split-KV, online softmax)
 *     out[b][h] = o~ . P_V[g]^T
 * which equals the definition up to rounding by associativity of the products,
 * (q . P_K) . K_down[t] = q . (K_down[t] . P_K^T) and
 * (sum_t p_t V_down[t]) . P_V^T = sum_t p_t (V_down[t] . P_V^T);
 * orthonormality of the bases is not needed for this.  The products run on the
 * tensor cores with fp32 accumulation; q~, the softmax weights and o~ enter them
 * as a bf16 pair (rounding plus rounded residual), about 16 significant bits.
 * L == 0 gives out = 0.  Rows at or beyond seq_lens[b] do not affect the result
 * (they may be fetched with a 32-row tile, and are masked and zeroed on chip).
 *
 *   q            : bf16 [B][Hq][d]
 *   P_K, P_V     : bf16 [Hkv][d][rK], [Hkv][d][rV]
 *   k_lat, v_lat : bf16 [B][Hkv][L_max][rK], [B][Hkv][L_max][rV]
 *   seq_lens     : int32 [B] on the device, each in [0, max_seq_len]; a length
 *                  outside that range sets STIEF_DEV_BAD_LENGTH in *dev_status
 *                  and gives out = 0 for that sequence
 *   out          : bf16 [B][Hq][d] (written)
 *   workspace    : device scratch of at least workspace_bytes >=
 *                  stief_decode_workspace_bytes(B, Hq, Hkv, rV, max_seq_len)
 *                  bytes.  Zero-fill it once before its first use: its ticket
 *                  counters and merge words must be zero when a call starts, and
 *                  every call that runs to completion leaves them at zero again,
 *                  so the same workspace serves any later call (any sizes) on the
 *                  same stream without clearing.  After a call whose dev_status
 *                  reports a timeout, zero it again
 *   max_seq_len  : host-side upper bound of seq_lens (<= L_max); sizes the grid
 *   num_splits   : 0 = automatic, otherwise the number of KV splits per sequence
 *                  (1 .. stief_decode_max_splits(max_seq_len))
 *
 * One kernel runs on `stream`, a CTA per (split, KV head, query sub-group,
 * sequence): query projection, scores, online softmax and latent value mix over
 * its token range; the splits of each (sequence, KV head, sub-group) are merged
 * (log-sum-exp) and up-projected once, through the workspace (see
 * stief_decode_workspace_bytes).  The merge that waits for the other splits' words
 * assumes every CTA of the grid can run at once, as on an otherwise idle GPU; a
 * kernel on another stream that holds SMs until this one finishes would make that
 * wait run out (STIEF_DEV_WAIT_TIMEOUT after 2 s).  The kernel is launched
 * as a programmatic dependent of the preceding work in the stream: it may be
 * scheduled while that work drains and reads no input before it has completed,
 * except P_K and the first tiles of k_lat and v_lat, which it requests first so
 * that their latency overlaps that work.  So if the kernel that immediately
 * precedes the call in the stream lets its dependents start early (programmatic
 * dependent launch), it must write neither P_K nor any row of k_lat or v_lat
 * below seq_lens[b] - 1; the row just below each length is read again after the
 * wait, so stief_append_decode calls may follow one another on the same caches.
 * This library's kernels never write the bases, and a decode call issued right after
 * one of its compress calls in the same stream reads no cache row before the wait
 * (the library keeps that note per stream).  The rule on P_K holds for every call
 * that takes it; the rule on the cache rows for every decode call, with two
 * differences: the _paged calls also read the block-table entries of their first
 * tiles before the wait (the preceding kernel must not write the entries of pages
 * that hold rows below seq_lens[b]), and the int8, 4-bit and joint-value calls read
 * no row again after the wait (the preceding kernel must write no row below
 * seq_lens[b], the row just below it included); a decode issued right after one of
 * this library's int8 fused steps in the same stream requests no cache row before its
 * wait (the library notes it per stream, as after a compress), so
 * stief_append_decode_q8 calls may follow one another.
 * Returns STIEF_OK or an argument error (nothing launched).
 */
STIEF_API stief_status stief_decode_attention(const uint16_t* q, const uint16_t* P_K,
                                    const uint16_t* P_V, const uint16_t* k_lat,
                                    const uint16_t* v_lat, const int32_t* seq_lens,
                                    uint16_t* out, void* workspace, size_t workspace_bytes,
                                    int B, int Hq, int Hkv, int d, int rK, int rV, int L_max,
                                    int max_seq_len, int num_splits,
                                    uint32_t* dev_status, stief_stream_t stream);

/*
 * stief_append_decode -- one whole decode step of the hot path in one kernel: the
 * append of stief_compress_append with T = 1 followed by stief_decode_attention over
 * the grown cache (StiefAttention technical summary, "Mecanismo Central" item 5:
 * keys and values are stored compressed, K_down = K P_K, V_down = V P_V, and
 * attention runs over their reconstructions).
 *
 * For every sequence b (L = seq_lens[b] on entry) and KV head g:
 *     k_lat[b][g][L] = bf16_RNE(k_new[b][g] . P_K[g])      (fp32 accumulation)
 *     v_lat[b][g][L] = bf16_RNE(v_new[b][g] . P_V[g])
 * then, for every query head h of g, out[b][h] is stief_decode_attention's result
 * over the L + 1 tokens [0, L], and seq_lens[b] = L + 1 once the kernel completes.
 * Rows other than L are not written.  If L + 1 > L_max the sequence is not appended
 * to (STIEF_DEV_CAPACITY_OVERFLOW is set, seq_lens[b] stays L) and out[b] attends over
 * the L tokens present; if L + 1 > max_seq_len, STIEF_DEV_BAD_LENGTH is set likewise.
 *
 *   k_new, v_new : bf16 [B][Hkv][d] (the new token's key and value rows)
 *   seq_lens     : int32 [B] on the device, read and then incremented
 *   max_seq_len  : host-side upper bound of the lengths after the append (<= L_max)
 *   other arguments as for stief_decode_attention (same workspace size and rules)
 *
 * The stored rows equal stief_compress_append's up to the order of the fp32 sums
 * (both round once to bf16).  The paper has no fused call: this one removes the two
 * extra kernel launches of the separate append from every step.
 * Returns STIEF_OK or an argument error (nothing launched).
 */
STIEF_API stief_status stief_append_decode(const uint16_t* q, const uint16_t* k_new,
                                 const uint16_t* v_new, const uint16_t* P_K,
                                 const uint16_t* P_V, uint16_t* k_lat, uint16_t* v_lat,
                                 int32_t* seq_lens, uint16_t* out, void* workspace,
                                 size_t workspace_bytes, int B, int Hq, int Hkv, int d, int rK,
                                 int rV, int L_max, int max_seq_len, int num_splits,
                                 uint32_t* dev_status, stief_stream_t stream);

/*
 * stief_decode_latent -- the decode step in the latent space only, for models whose
 * attention weights absorb the bases (StiefAttention technical summary, "Mecanismo
 * Central" item 5, last sentence: the projection bases can be folded into the
 * attention's linear weights, at no extra run time over standard low-rank methods).
 * With W_Q P_K as the query weight and P_V^T W_O as the output weight, the model
 * hands over q~ directly and consumes o~; the query projection and the up-projection
 * of stief_decode_attention drop out.
 *
 * For every sequence b and query head h (KV head g = h / (Hq/Hkv), L = seq_lens[b]):
 *     s_t = q_lat[b][h] . k_lat[b][g][t] / sqrt(d)          t < L
 *     out_lat[b][h] = bf16_RNE( sum_t softmax(s)_t v_lat[b][g][t] )
 * i.e. stief_decode_attention with q~ given and o~ returned: for q_lat = q . P_K,
 * out_lat . P_V^T equals stief_decode_attention's output up to rounding (q~ enters
 * here as bf16, there as fp32).  Same split-KV online softmax, precision (q~, the
 * softmax weights and o~ enter the tensor-core products as bf16 pairs, fp32
 * accumulation), masking and L == 0 behaviour.
 *
 *   q_lat        : bf16 [B][Hq][rK]
 *   k_lat, v_lat : bf16 [B][Hkv][L_max][rK], [B][Hkv][L_max][rV] (only read)
 *   out_lat      : bf16 [B][Hq][rV] (written)
 *   d            : the head dimension; sets the score scale 1/sqrt(d) (d == 128)
 *   seq_lens, workspace, max_seq_len, num_splits, dev_status, stream: as for
 *                  stief_decode_attention (same workspace size and rules)
 *
 * One kernel, as stief_decode_attention's without the base loads.
 * Returns STIEF_OK or an argument error (nothing launched).
 */
STIEF_API stief_status stief_decode_latent(const uint16_t* q_lat, const uint16_t* k_lat,
                                 const uint16_t* v_lat, const int32_t* seq_lens,
                                 uint16_t* out_lat, void* workspace, size_t workspace_bytes,
                                 int B, int Hq, int Hkv, int d, int rK, int rV, int L_max,
                                 int max_seq_len, int num_splits, uint32_t* dev_status,
                                 stief_stream_t stream);

/*
 * Paged latent caches (serving-style block tables).  StiefAttention's pages give no
 * memory layout; the idea of fixed-size token blocks for regular, coalesced cache access
 * comes from a neighbouring method's page (HyLRA technical summary, section 2.4,
 * "hardware-efficient optimisations": block-level sparsity over fixed token blocks).
 * This library's paged form keeps each cache as a pool of pages,
 *     k_pages : bf16 [num_pages][Hkv][page_size][rK]
 *     v_pages : bf16 [num_pages][Hkv][page_size][rV]
 * and gives every sequence b a row of the block table,
 *     block_table : int32 [B][max_pages] (device), page ids in [0, num_pages),
 * so that token t of (b, KV head h) is row t % page_size of page block_table[b][t /
 * page_size], head h.  A sequence's capacity is max_pages * page_size tokens (the
 * contiguous calls' L_max).  page_size is a multiple of 64 (>= 64); num_pages *
 * Hkv * page_size < 2^31.  Entries for pages the sequence does not reach are never
 * read for its tokens.  An append whose new rows need a page with an id outside
 * [0, num_pages) (or past max_pages) is refused for that sequence as a full cache is:
 * STIEF_DEV_CAPACITY_OVERFLOW, nothing written, the length unchanged.  A decode never
 * checks the pages below the length (they read as zeros if unmapped, which masks
 * nothing): the caller maps every page below the length.  block_table must be 4-byte
 * aligned; the pools 16-byte.
 * The calls below are their contiguous counterparts with k_lat / v_lat replaced by
 * the pools and L_max by (num_pages, page_size, max_pages); everything else --
 * results, workspace, status words, launch behaviour -- is the same.
 */
STIEF_API stief_status stief_compress_append_paged(const uint16_t* k_new, const uint16_t* v_new,
                                         const uint16_t* P_K, const uint16_t* P_V,
                                         uint16_t* k_pages, uint16_t* v_pages,
                                         const int32_t* block_table, int32_t* seq_lens, int B,
                                         int Hkv, int T, int d, int rK, int rV, int num_pages,
                                         int page_size, int max_pages, uint32_t* dev_status,
                                         stief_stream_t stream);

STIEF_API stief_status stief_decode_attention_paged(const uint16_t* q, const uint16_t* P_K,
                                          const uint16_t* P_V, const uint16_t* k_pages,
                                          const uint16_t* v_pages, const int32_t* block_table,
                                          const int32_t* seq_lens, uint16_t* out, void* workspace,
                                          size_t workspace_bytes, int B, int Hq, int Hkv, int d,
                                          int rK, int rV, int num_pages, int page_size,
                                          int max_pages, int max_seq_len, int num_splits,
                                          uint32_t* dev_status, stief_stream_t stream);

STIEF_API stief_status stief_append_decode_paged(const uint16_t* q, const uint16_t* k_new,
                                       const uint16_t* v_new, const uint16_t* P_K,
                                       const uint16_t* P_V, uint16_t* k_pages, uint16_t* v_pages,
                                       const int32_t* block_table, int32_t* seq_lens,
                                       uint16_t* out, void* workspace, size_t workspace_bytes,
                                       int B, int Hq, int Hkv, int d, int rK, int rV,
                                       int num_pages, int page_size, int max_pages,
                                       int max_seq_len, int num_splits, uint32_t* dev_status,
                                       stief_stream_t stream);

/*
 * int8 latent caches (the low-bit form).  The pages report the compressed cache to be
 * robust to 4- and 8-bit quantisation (StiefAttention technical summary, "Resultados
 * Experimentais", the quantisation-compatibility result) but fix no scheme; this library
 * stores each latent
 * row (one token, one KV head) as int8 codes and one fp32 scale:
 *     k_q : int8 [B][Hkv][L_max][rK],  k_s : float [B][Hkv][L_max]  (likewise v_q, v_s)
 *     scale = max_c |x_c| / 127,  code_c = RNE(x_c / scale) in [-127, 127]
 * where x is the row rounded to bf16 (what the bf16 cache would hold), both divisions in
 * IEEE fp32; a zero row is scale 0 and codes 0.  A value stands for code * scale.
 * A row takes r + 4 bytes instead of the bf16 cache's 2 r.  L_max must be a multiple of 64; k_s, v_s, k_q, v_q
 * 16-byte aligned.  The calls are their bf16 counterparts on this form: the compress writes
 * codes and scales; the decode attends over code * scale.  On chip the codes enter the integer
 * tensor-core MMA as they are: q~ is held per head as 16-bit fixed point (relative step
 * 2^-15 of its largest element) and each tile's softmax weights per head as 16-bit fixed point
 * of the tile's largest weight, each split into two 8-bit parts, so both products are exact
 * in 32-bit integers; the row scales multiply the scores and the weights.  Paged int8 caches
 * are the _q8_paged calls below.  stief_append_decode_q8 is the fused step on this form: one
 * kernel appends the new token (its projected rows rounded to bf16, then quantised exactly as
 * the compress does: codes into k_q / v_q and scales into k_s / v_s at row seq_lens[b]) and
 * decodes over the grown cache, with stief_append_decode's launch behaviour and rules; it is
 * not provided for 4-bit or paged int8 caches.
 */
STIEF_API stief_status stief_compress_append_q8(const uint16_t* k_new, const uint16_t* v_new,
                                      const uint16_t* P_K, const uint16_t* P_V, int8_t* k_q,
                                      int8_t* v_q, float* k_s, float* v_s, int32_t* seq_lens,
                                      int B, int Hkv, int T, int d, int rK, int rV, int L_max,
                                      uint32_t* dev_status, stief_stream_t stream);

STIEF_API stief_status stief_decode_attention_q8(const uint16_t* q, const uint16_t* P_K,
                                       const uint16_t* P_V, const int8_t* k_q, const int8_t* v_q,
                                       const float* k_s, const float* v_s,
                                       const int32_t* seq_lens, uint16_t* out, void* workspace,
                                       size_t workspace_bytes, int B, int Hq, int Hkv, int d,
                                       int rK, int rV, int L_max, int max_seq_len,
                                       int num_splits, uint32_t* dev_status,
                                       stief_stream_t stream);

STIEF_API stief_status stief_append_decode_q8(const uint16_t* q, const uint16_t* k_new,
                                    const uint16_t* v_new, const uint16_t* P_K,
                                    const uint16_t* P_V, int8_t* k_q, int8_t* v_q, float* k_s,
                                    float* v_s, int32_t* seq_lens, uint16_t* out, void* workspace,
                                    size_t workspace_bytes, int B, int Hq, int Hkv, int d, int rK,
                                    int rV, int L_max, int max_seq_len, int num_splits,
                                    uint32_t* dev_status, stief_stream_t stream);

/*
 * int8 caches in page pools: the int8 form above with the paged layout of the _paged calls.
 *     k_pages : int8 [num_pages][Hkv][page_size][rK],  k_s_pages : float [num_pages][Hkv][page_size]
 * (likewise v_pages, v_s_pages): token t of (sequence b, KV head h) is row t % page_size of page
 * block_table[b][t / page_size], head h, in both the code and the scale pools.  page_size a
 * multiple of 64; the capacity is max_pages * page_size.  Everything else is as for the
 * _paged and _q8 calls.
 */
STIEF_API stief_status stief_compress_append_q8_paged(const uint16_t* k_new, const uint16_t* v_new,
                                            const uint16_t* P_K, const uint16_t* P_V,
                                            int8_t* k_pages, int8_t* v_pages, float* k_s_pages,
                                            float* v_s_pages, const int32_t* block_table,
                                            int32_t* seq_lens, int B, int Hkv, int T, int d,
                                            int rK, int rV, int num_pages, int page_size,
                                            int max_pages, uint32_t* dev_status,
                                            stief_stream_t stream);

STIEF_API stief_status stief_decode_attention_q8_paged(const uint16_t* q, const uint16_t* P_K,
                                             const uint16_t* P_V, const int8_t* k_pages,
                                             const int8_t* v_pages, const float* k_s_pages,
                                             const float* v_s_pages, const int32_t* block_table,
                                             const int32_t* seq_lens, uint16_t* out,
                                             void* workspace, size_t workspace_bytes, int B,
                                             int Hq, int Hkv, int d, int rK, int rV, int num_pages,
                                             int page_size, int max_pages, int max_seq_len,
                                             int num_splits, uint32_t* dev_status,
                                             stief_stream_t stream);

/*
 * 4-bit latent caches (the pages' other quantisation width; same per-row reading as the int8
 * form): each latent row (one token, one KV head) as symmetric 4-bit codes and one fp32 scale,
 *     scale = max_c |x_c| / 7,  code_c = RNE(x_c / scale) in [-7, 7]
 * (x the bf16-rounded row, both divisions in IEEE fp32; a zero row is scale 0, codes 0), two
 * codes per byte, column 2j in the low nibble of byte j (4-bit two's complement):
 *     k_q : uint8 [B][Hkv][L_max][rK / 2],  k_s : float [B][Hkv][L_max]  (likewise v_q, v_s)
 * A row takes r / 2 + 4 bytes.  rK and rV must be multiples of 32 (rows of whole 16-byte
 * units), L_max a multiple of 64; k_s, v_s, k_q, v_q 16-byte aligned.  The calls are the int8
 * ones on this form: the compress writes codes and scales; the decode attends over
 * code * scale, the codes entering the integer MMA as 16 x code (each byte's nibbles moved to
 * the top of a byte), q~ and the weights as 16-bit fixed point in two 8-bit parts as for the
 * int8 form.  Paged 4-bit caches and the fused step are not provided.
 */
STIEF_API stief_status stief_compress_append_q4(const uint16_t* k_new, const uint16_t* v_new,
                                      const uint16_t* P_K, const uint16_t* P_V, uint8_t* k_q,
                                      uint8_t* v_q, float* k_s, float* v_s, int32_t* seq_lens,
                                      int B, int Hkv, int T, int d, int rK, int rV, int L_max,
                                      uint32_t* dev_status, stief_stream_t stream);

STIEF_API stief_status stief_decode_attention_q4(const uint16_t* q, const uint16_t* P_K,
                                       const uint16_t* P_V, const uint8_t* k_q, const uint8_t* v_q,
                                       const float* k_s, const float* v_s,
                                       const int32_t* seq_lens, uint16_t* out, void* workspace,
                                       size_t workspace_bytes, int B, int Hq, int Hkv, int d,
                                       int rK, int rV, int L_max, int max_seq_len,
                                       int num_splits, uint32_t* dev_status,
                                       stief_stream_t stream);

/*
 * Joint value latents (STAR-KV technical summary, "Metodologia" item 2, the hybrid
 * decomposition: keys keep one basis per KV head, the values of all KV heads are factored
 * together, and the value reconstruction is absorbed into the output projection).  The values
 * of a token's Hkv heads, concatenated head 0 first, are projected by one basis
 *     P_VJ : bf16 [Hkv*d][rV]
 * and the cache holds one value latent per token, shared by every KV head:
 *     v_joint : bf16 [B][L_max][rV]
 * KV head g's values are rebuilt from rows [g*d, (g+1)*d) of P_VJ, so P_VJ read as
 * [Hkv][d][rV] has the per-head P_V layout.  The keys, queries, outputs, workspace, status
 * words and launch behaviour are those of the per-head calls:
 *   stief_decode_attention_joint_v: stief_decode_attention with v_lat -> v_joint and
 *       P_V -> P_VJ:  o_h = (sum_t p_t v_joint[t]) . (rows of KV head g of P_VJ)^T;
 *   stief_decode_latent_joint_v: stief_decode_latent with v_lat -> v_joint:
 *       o~_h = sum_t p_t v_joint[t];
 *   stief_compress_append_joint_v: stief_compress_append with the values projected jointly,
 *       v_joint[b][seq_lens[b] + t] = bf16_RNE( [v_new[b][0][t] | ... | v_new[b][Hkv-1][t]] . P_VJ )
 *       (fp32 accumulation), keys per head as in stief_compress_append, then
 *       seq_lens[b] += T; the same skipping and status bits for a full cache or a bad length.
 *       T >= 128 runs on the tensor cores when the joint basis (half of it per CTA when an
 *       even Hkv lets the value tiles be split over CTA pairs, with a 512 * rV-byte exchange
 *       area) and two 32 KB input stages fit one CTA's shared memory (e.g. Hkv = 8: rV <= 96;
 *       Hkv = 4: rV <= 128), with the launch behaviour of
 *       stief_compress_append's tensor-core path (a decode issued next on the same stream
 *       waits for it before reading any cache tile); otherwise CUDA cores.  B <= 65535.
 * The key cache has the per-head limits (B * Hkv * L_max < 2^31).  No fused append, paged or
 * int8 form.
 */
STIEF_API stief_status stief_compress_append_joint_v(
    const uint16_t* k_new, const uint16_t* v_new, const uint16_t* P_K, const uint16_t* P_VJ,
    uint16_t* k_lat, uint16_t* v_joint, int32_t* seq_lens, int B, int Hkv, int T, int d, int rK,
    int rV, int L_max, uint32_t* dev_status, stief_stream_t stream);

STIEF_API stief_status stief_decode_attention_joint_v(
    const uint16_t* q, const uint16_t* P_K, const uint16_t* P_VJ, const uint16_t* k_lat,
    const uint16_t* v_joint, const int32_t* seq_lens, uint16_t* out, void* workspace,
    size_t workspace_bytes, int B, int Hq, int Hkv, int d, int rK, int rV, int L_max,
    int max_seq_len, int num_splits, uint32_t* dev_status, stief_stream_t stream);

STIEF_API stief_status stief_decode_latent_joint_v(
    const uint16_t* q_lat, const uint16_t* k_lat, const uint16_t* v_joint,
    const int32_t* seq_lens, uint16_t* out_lat, void* workspace, size_t workspace_bytes, int B,
    int Hq, int Hkv, int d, int rK, int rV, int L_max, int max_seq_len, int num_splits,
    uint32_t* dev_status, stief_stream_t stream);

/*
 * stief_decode_attention_noalloc -- stief_decode_attention without a workspace
 * argument and without any device allocation.  The paper has no counterpart: this
 * is a deployment variant for callers that cannot obtain device memory when they
 * decode (a serving engine whose KV-cache pool already holds nearly all of HBM, a
 * host framework whose operator interface passes only inputs and outputs, a
 * latency-critical loop that must not call cudaMalloc).
 *
 * Same arguments, meaning and result as stief_decode_attention, minus
 * workspace / workspace_bytes.  The per-split partial states live in a fixed 8 MiB
 * array of device memory owned by the library (one per GPU that loads it, held
 * until the process exits).  Sizes whose partial states, for the split count
 * actually used, exceed 8 MiB -- B*Hkv*ceil(G/G_T)*G_T*splits*(d+2)*8 bytes with
 * G = Hq/Hkv and G_T the smallest of 1, 2, 4, 8 that is >= min(G, 8) -- plus the
 * ticket counters, return
 * STIEF_ERR_WORKSPACE and launch nothing.  The first call on each device looks up
 * the array's device address (cudaGetSymbolAddress) with that device current; make
 * that first call before any stream capture.  All calls on a device share the
 * array: calls whose kernels overlap on the GPU race on it, so the caller must
 * order them (e.g. one stream).  The array keeps the last call's contents.  Its
 * ticket counters and merge words must be zero when a kernel starts; a call that
 * stopped early (STIEF_DEV_WAIT_TIMEOUT) may leave them otherwise, and the caller
 * cannot reach the array, so every call zeroes the part it uses with
 * cudaMemsetAsync on `stream` before its launch (a memset, not an allocation).
 * Calls no cudaMalloc, cudaFree or allocating library routine.
 */
STIEF_API stief_status stief_decode_attention_noalloc(
    const uint16_t* q, const uint16_t* P_K, const uint16_t* P_V, const uint16_t* k_lat,
    const uint16_t* v_lat, const int32_t* seq_lens, uint16_t* out, int B, int Hq, int Hkv, int d,
    int rK, int rV, int L_max, int max_seq_len, int num_splits, uint32_t* dev_status,
    stief_stream_t stream);

/*
 * stief_read_device_status -- synchronises `stream`, copies the device status
 * word to *value, and returns STIEF_OK if it is zero, STIEF_ERR_DEVICE_STATUS
 * if not, STIEF_ERR_CUDA if the copy failed, STIEF_ERR_INVALID_ARG for NULLs.
 */
STIEF_API stief_status stief_read_device_status(const uint32_t* dev_status, uint32_t* value,
                                      stief_stream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
STIEF_API const char* stief_status_string(stief_status status);

#ifdef __cplusplus
}
#endif

#endif /* STIEF_H */
