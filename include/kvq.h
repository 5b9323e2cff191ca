/*
 * kvq.h - C ABI of the rotated-angle KV-cache codec and of decode attention
 * over the compressed cache, for NVIDIA B200 (sm_100a).
 *
 * Method: "TurboAngle: Near-Lossless KV Cache Compression via Uniform Angle
 * Quantization", Abstract.  Each key or value head vector is multiplied by a
 * seeded random +-1 diagonal D, transformed by the Fast Walsh-Hadamard
 * transform H (scaled by 1/sqrt(d)), split into consecutive element pairs,
 * and every pair is stored as a uniformly quantized angle plus a quantized
 * norm: 8-bit linear norms for keys, 4-bit log-space norms for values, with
 * the codebook size L chosen per layer and separately for K and V
 * ("per-layer early-boost").  Decode attention reads the codes directly and
 * never materialises a dequantized cache (the on-the-fly reconstruction
 * principle of "OCTOPUS: Joint Triplet Quantization for KV Cache via
 * Octahedral Parametrization", sections "TL;DR" and "Why it matters").
 *
 * The pages give the method in words only.  This header fixes every formula
 * and byte the library uses; where the pages are silent the plainest reading
 * is taken and marked "(reading)".
 *
 * ---------------------------------------------------------------------------
 * Definitions (d = head_dim, P = d/2 pairs, b = angle bits)
 * ---------------------------------------------------------------------------
 *   H      Sylvester-ordered Hadamard matrix, H[j][k] = (-1)^popcount(j & k)
 *          (reading: natural order; H*H = d*I).
 *   D      diagonal of signs s[k] in {+1,-1}, one vector per (layer, K|V),
 *          passed in as data (int8, values +1 / -1).
 *   z      = H * D * x / sqrt(d)                        (rotation, x fp16)
 *   r_i    = |(z[2i], z[2i+1])|,  theta_i = atan2(z[2i+1], z[2i])
 *   a_i    = floor((theta_i + pi) * L / (2 pi)) mod L   (uniform angle code;
 *            a pair that is exactly (0,0) gets a_i = 0 (reading))
 *   b      = smallest integer >= 1 with 2^b >= L        (bits per angle code)
 *   Reconstruction angle (reading: bin centre, so |theta - theta^| <= pi/L):
 *          theta^_a = -pi + (a + 1/2) * 2 pi / L
 *
 *   Norm modes (per codec):
 *   KVQ_NORM_LIN8  M = fp16(max_i r_i) (round to nearest even; saturates to
 *                  65504; reading), c_i = min(255, floor(255 r_i / M + 1/2)),
 *                  all c_i = 0 when M = 0.  r^_i = c_i * M / 255.
 *   KVQ_NORM_LOG4  l_i = log2(max(r_i, 2^-24)), LO = fp16(min_i l_i),
 *                  HI = fp16(max_i l_i),
 *                  c_i = clamp(floor(15 (l_i - LO) / (HI - LO) + 1/2), 0, 15),
 *                  all c_i = 0 when HI = LO.
 *                  r^_i = 2^(LO + c_i (HI - LO) / 15).
 *   (round-half-up and the 2^-24 floor are readings.)
 *
 *   Dequantized vector: z^[2i] = r^_i cos theta^_i, z^[2i+1] = r^_i sin theta^_i,
 *                       x^ = D * H * z^ / sqrt(d)   (the exact inverse rotation).
 *
 *   Decode attention for query head h (GQA: KV head = h / (H_q / H_kv),
 *   reading: the usual grouped-query convention):
 *     q'       = H * D_K * q / sqrt(d)                  (once per head)
 *     s_t      = tau * sum_i r^K_{t,i} (q'[2i] cos theta^K_{t,i} + q'[2i+1] sin theta^K_{t,i})
 *              (= tau * q . k^_t, because H*D/sqrt(d) is orthogonal)
 *     p_t      = softmax_t(s_t) over t < ctx_len[b]  (no mask inside the range)
 *     acc      = sum_t p_t z^V_t                        (rotated domain)
 *     out      = D_V * H * acc / sqrt(d)                (one inverse FWHT per head)
 *   tau is the softmax_scale argument (1/sqrt(d) is the usual choice).
 *
 * ---------------------------------------------------------------------------
 * Packed layout of the compressed cache (one "plane" per K or V per layer)
 * ---------------------------------------------------------------------------
 * A plane is three caller-owned device arrays, each laid out
 * [B][H_kv][capacity][row], row sizes from kvq_row_bytes():
 *   angles  ceil(P*b/32) 32-bit little-endian words per token; code i lives in
 *           bits [i*b, i*b + b) of the row's bit stream, where bit k of word w
 *           is stream bit 32w + k (LSB first).
 *   norms   LIN8: P bytes, byte i = c_i.
 *           LOG4: P/2 bytes, byte j = c_{2j} | c_{2j+1} << 4.
 *   params  LIN8: one IEEE fp16 M (2 bytes).  LOG4: fp16 LO then fp16 HI
 *           (4 bytes).  A zero parameter is stored as +0 (reading).
 * Requirements checked by every call: capacity % 16 == 0; every array
 * 16-byte aligned.  Token t of sequence (b, h) is row (b*H_kv + h)*capacity + t.
 *
 * ---------------------------------------------------------------------------
 * Conventions
 * ---------------------------------------------------------------------------
 * Ownership: all memory is owned by the caller.  The library never allocates
 *   or frees device memory; scratch space is passed in (workspace).
 * Execution: every compute call is asynchronous on `stream` (a cudaStream_t,
 *   passed as void*; NULL = legacy default stream).
 * Errors: invalid arguments return KVQ_EINVAL or KVQ_EUNSUPPORTED before any
 *   launch; a failed launch returns KVQ_ECUDA.  The message for the last
 *   non-OK status of the calling thread is kvq_last_error().  Conditions seen
 *   on the device (a ctx_len outside [0, capacity], a bounded wait that ran
 *   out) are OR-ed into *err_word (KVQ_DEVERR_* bits) when err_word is not
 *   NULL; the kernels never trap.
 * Inputs must be finite; NaN or Inf inputs give unspecified codes.
 *
 * Environment: KVQ_DEBUG (set, not "0") makes every decode call first check
 * the cache rows it reads (tokens 0 .. ctx_len[b]-1) for values the encoder
 * never writes and report them as KVQ_DEVERR_BAD_CODE in err_word; it costs a
 * second read of the cache and is meant for debugging.  KVQ_PROFILE (set, not
 * "0") brackets the launches of every call with an NVTX range named after the
 * call, for profilers.  Both are read once, at the first call.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KVQ_OK = 0,
    KVQ_EINVAL = -1,       /* argument out of range, misaligned or NULL    */
    KVQ_EUNSUPPORTED = -2, /* valid for the codec, not built into kernels  */
    KVQ_ECUDA = -3,        /* CUDA runtime reported an error on launch     */
    KVQ_ETIMEOUT = -4      /* reserved: a device-side bounded wait expired */
} kvq_status;

typedef enum { KVQ_NORM_LIN8 = 0, KVQ_NORM_LOG4 = 1 } kvq_norm_mode;

/* Device error bits OR-ed into *err_word. */
#define KVQ_DEVERR_CTX_RANGE 0x1  /* ctx_len[b] < 0 or > capacity: clipped   */
#define KVQ_DEVERR_TIMEOUT 0x2    /* an mbarrier wait hit its iteration cap  */
#define KVQ_DEVERR_PAGE_RANGE 0x4 /* a page-table entry outside [0, num_pages):
                                     page 0 was read or written instead       */
#define KVQ_DEVERR_BAD_CODE 0x8   /* KVQ_DEBUG checks: a cache row holds a value
                                     the encoder never writes (an angle code
                                     >= L, a non-finite fp16 parameter, LOG4
                                     HI < LO, LIN8 M < 0)                    */

/* One codec: per layer and separately for K and V ("per-layer early-boost").
 * head_dim: power of two, 4..256.  L: 2..65536.  Every call takes every
 * codec (decode: either norm mode for K and for V). */
typedef struct {
    int32_t head_dim;
    int32_t L;
    int32_t norm_mode; /* kvq_norm_mode */
} kvq_codec;

/* One compressed plane (see "Packed layout").  Pointers are device pointers
 * owned by the caller; capacity is tokens per (batch, KV head). */
typedef struct {
    void* angles;
    void* norms;
    void* params;
    int64_t capacity;
} kvq_plane;

/* A paged plane: the rows of all sequences live in fixed-size pages of one
 * shared pool, found through a page table (a serving cache that grows each
 * sequence page by page; the TurboAngle page stores no cache layout of its
 * own, this one keeps its row format and only moves rows between pages).
 *   angles, norms, params  device pools laid out [num_pages][H_kv][page_tokens][row]
 *                          (rows as in "Packed layout"), 16-byte aligned
 *   pages        device int32 [B][max_pages]: pages[b][i] holds tokens
 *                i*page_tokens .. (i+1)*page_tokens - 1 of sequence b, all KV heads
 *   page_tokens  tokens per page: a positive multiple of 128 (one page holds
 *                whole staged tiles of the decode kernel)
 *   max_pages    entries per sequence in `pages`; the capacity of every
 *                sequence is max_pages * page_tokens
 *   num_pages    pages in the pool; an entry outside [0, num_pages) that a
 *                call reaches is replaced by page 0 and sets KVQ_DEVERR_PAGE_RANGE
 * Token t of sequence (b, h) is row (pages[b][t / page_tokens]*H_kv + h)
 * * page_tokens + t % page_tokens of each pool.  K and V may share a table. */
typedef struct {
    void* angles;
    void* norms;
    void* params;
    const int32_t* pages;
    int32_t page_tokens;
    int32_t max_pages;
    int64_t num_pages;
} kvq_paged_plane;

/* Bytes per token of one plane array: which = 0 angles, 1 norms, 2 params.
 * Returns a negative kvq_status for an invalid codec or `which`.  Host only. */
int64_t kvq_row_bytes(const kvq_codec* codec, int32_t which);

/* Bits per angle code for codebook size L (smallest b >= 1 with 2^b >= L);
 * negative for L outside 2..65536.  Host only. */
int32_t kvq_angle_bits(int32_t L);

/* Encode (prefill when T > 1, append when T == 1).
 * Follows the encode steps of the TurboAngle abstract (random diagonal, FWHT
 * domain, consecutive pairs, uniform angles, 8-bit / 4-bit log norms).
 *   signs  device int8 [head_dim], +1 / -1 (the diagonal D of this layer/K|V)
 *   x      device fp16 [B][H_kv][T][head_dim], contiguous, 16-byte aligned
 *   out    plane receiving tokens pos0 .. pos0+T-1 of every (b, h);
 *          requires 0 <= pos0 and pos0 + T <= out->capacity.
 * Codes are bit-exact to the definitions above except where a value lies
 * within floating-point error of a decision edge of the definition (there
 * the kernel re-decides from the exactly computed rotation in fp64).
 * T == 0 is a no-op. */
int kvq_encode(const kvq_codec* codec, const int8_t* signs, const void* x,
               int32_t B, int32_t H_kv, int32_t T, int64_t pos0,
               const kvq_plane* out, void* stream);

/* Encode the same token range of a layer's K and V in one launch: the same
 * result as kvq_encode(kc, signs_k, k, B, H_kv, T, pos0, K) followed by
 * kvq_encode(vc, signs_v, v, B, H_kv, T, pos0, V).  The per-token append of
 * a decode step writes one K and one V row per (b, h); one launch instead of
 * two halves the fixed cost of that step (the TurboAngle abstract encodes K
 * and V independently, so nothing ties the two halves together but the
 * launch).  Requires kc->head_dim == vc->head_dim; the codecs may differ in
 * L and norm mode.  Arguments as for kvq_encode; argument errors are
 * reported before anything is launched.  T == 0 is a no-op. */
int kvq_encode_kv(const kvq_codec* kc, const int8_t* signs_k, const void* k,
                  const kvq_plane* K, const kvq_codec* vc, const int8_t* signs_v,
                  const void* v, const kvq_plane* V, int32_t B, int32_t H_kv,
                  int32_t T, int64_t pos0, void* stream);

/* Dequantize tokens pos0 .. pos0+T-1 of a plane back to fp16: the
 * reconstruction of the TurboAngle abstract's codec (each pair's norm from
 * its norm code, its angle the centre of its bin, then the inverse of the
 * random rotation), x^ = D H z^ / sqrt(d) as defined above.
 *   y  device fp16 [B][H_kv][T][head_dim], 16-byte aligned, caller-owned.
 * Arguments are checked as for kvq_encode; T == 0 is a no-op. */
int kvq_dequant(const kvq_codec* codec, const int8_t* signs,
                const kvq_plane* in, int32_t B, int32_t H_kv, int32_t T,
                int64_t pos0, void* y, void* stream);

/* Split count the library would choose for a decode launch (host logic,
 * deterministic).  Its cost model: one CTA per SM, a CTA's time is its
 * ceil(max_ctx / splits) tokens plus a fixed cost of about 512 tokens'
 * worth (prologue, first copy, merge, combine); the split count minimises
 * waves x (tokens per CTA + 512) over at most eight waves on sm_count SMs,
 * the fewer CTAs on ties.  At least 1, at most ceil(max_ctx / 128). */
int32_t kvq_decode_num_splits(int32_t B, int32_t H_kv, int64_t max_ctx,
                              int32_t sm_count);

/* Workspace bytes kvq_decode_attn needs for `num_splits` splits: B*H_q int32
 * completion counters (rounded up to 16 bytes), then per (b, query head,
 * split) an fp32 running max and softmax denominator, then an fp32
 * [head_dim] partial accumulator (rotated domain). */
int64_t kvq_decode_workspace_bytes(int32_t B, int32_t H_q, int32_t head_dim,
                                   int32_t num_splits);

/* Split-K decode attention over the compressed cache, one layer, one new
 * query per sequence: attention scores read straight from the codes, never
 * from a dequantized cache (TurboAngle abstract for the codec; the
 * on-the-fly reconstruction principle of the OCTOPUS page, "TL;DR" and "Why
 * it matters"), with the formulas of "Decode attention" above.
 *   q          device fp16 [B][H_q][head_dim]
 *   kc, vc     K and V codecs (same head_dim, any L and norm modes; head_dim
 *              64/128, G 1/2/4/8, L <= 256 with LIN8 K and LOG4 V run in the
 *              staged kernel, every other codec in the generic kernel)
 *   signs_k/v  device int8 [head_dim] diagonals used when K / V were encoded
 *   K, V       planes holding the cache; tokens 0 .. ctx_len[b]-1 are read
 *   ctx_len    device int32 [B]; values are clipped to [0, min(max_ctx,
 *              capacity)] and a clip sets KVQ_DEVERR_CTX_RANGE
 *   max_ctx    host upper bound of ctx_len used to size the splits (>= 0)
 *   softmax_scale  tau
 *   num_splits >= 1 (kvq_decode_num_splits gives the default)
 *   workspace  device scratch of ws_bytes >= kvq_decode_workspace_bytes(),
 *              16-byte aligned, zero-filled before its first use (every call
 *              leaves its counters at zero again); calls that share a
 *              workspace must be stream-ordered
 *   err_word   device int32 or NULL (see Errors)
 *   out        device [B][H_q][head_dim], fp16 (out_dtype 0) or fp32 (1);
 *              a sequence with ctx_len 0 gets zeros.
 * One kernel runs on `stream`: each CTA handles one (split, KV head, batch
 * entry); the last CTA of a (batch entry, KV head) to finish merges the
 * per-split softmax states, applies the inverse FWHT and D_V / sqrt(d) and
 * writes the output.  When num_splits <= 16 and every (batch entry, KV head)
 * cluster of num_splits CTAs fits on the GPU at once, the splits of each
 * (batch entry, KV head) run as one thread-block cluster instead and merge
 * through distributed shared memory; the workspace is then not touched
 * (it must still be passed). */
int kvq_decode_attn(const void* q, const kvq_codec* kc, const kvq_codec* vc,
                    const int8_t* signs_k, const int8_t* signs_v,
                    const kvq_plane* K, const kvq_plane* V,
                    const int32_t* ctx_len, int32_t B, int32_t H_q,
                    int32_t H_kv, int64_t max_ctx, float softmax_scale,
                    int32_t num_splits, void* workspace, int64_t ws_bytes,
                    int32_t* err_word, void* out, int32_t out_dtype,
                    void* stream);

/* Context-sharded decode, part 1: kvq_decode_attn over the tokens this GPU
 * holds, stopped before the combine.  When a sequence's cached context is
 * spread over several GPUs (each plane holding a range of its tokens, its own
 * ctx_len counting the tokens held here), each GPU runs this call on its
 * planes; the workspace then holds, at the offsets that
 * kvq_decode_workspace_bytes describes, per (b, query head, split) the
 * running maximum m (log2 units: the scores times softmax_scale times log2 e,
 * -inf for a split with no token), the denominator l = sum 2^(s - m) and the
 * accumulator sum 2^(s - m) z^_V in the rotated domain.  These are the
 * partials of the split combine that kvq_decode_attn performs (the softmax
 * and value formulas of "Decode attention" above); merging them across GPUs
 * gives the same result.  Arguments and checks as for kvq_decode_attn, with
 * no output; the completion counters are not touched.  All GPUs of one merge
 * use the same B, H_q, head_dim and num_splits. */
int kvq_decode_attn_partials(const void* q, const kvq_codec* kc,
                             const kvq_codec* vc, const int8_t* signs_k,
                             const int8_t* signs_v, const kvq_plane* K,
                             const kvq_plane* V, const int32_t* ctx_len,
                             int32_t B, int32_t H_q, int32_t H_kv,
                             int64_t max_ctx, float softmax_scale,
                             int32_t num_splits, void* workspace,
                             int64_t ws_bytes, int32_t* err_word,
                             void* stream);

/* Context-sharded decode, part 2: merge the partials of n_parts workspaces
 * (each kvq_decode_workspace_bytes(B, H_q, head_dim, num_splits) bytes, laid
 * out back to back in `parts`, e.g. after an all-gather) into the attention
 * output: M = max m, L = sum l 2^(m - M), z = sum acc 2^(m - M) / L over
 * every part and split, then o = D_V H z / sqrt(d), as the single-GPU
 * combine does.
 *   parts    device, 16-byte aligned, n_parts x workspace bytes
 *   signs_v  device int8 [head_dim], the V diagonal
 *   out      device fp16 or fp32 [B][H_q][head_dim]
 * head_dim a power of two in 4..256; 1 <= n_parts <= 4096 with n_parts x
 * num_splits <= 16384; a (b, head) whose parts hold no token gives 0. */
int kvq_decode_merge_partials(const void* parts, int32_t n_parts, int32_t B,
                              int32_t H_q, int32_t head_dim,
                              int32_t num_splits, const int8_t* signs_v,
                              void* out, int32_t out_dtype, void* stream);

/* One decode step of one layer, normally in one kernel: the append of each
 * sequence's new token fused into kvq_decode_attn.  For every b with 1 <= ctx_len[b]
 * <= min(max_ctx, capacity), the token at position ctx_len[b] - 1 of every
 * KV head is first written as
 *   kvq_encode_kv(kc, signs_k, k_new[b], K, vc, signs_v, v_new[b], V, ...)
 * would write it (same codes, byte for byte), then attention runs over
 * positions 0 .. ctx_len[b] - 1, the new token included, exactly as
 * kvq_decode_attn.  The TurboAngle abstract encodes K and V on arrival and
 * attends from codes; doing both in one launch is this library's choice:
 * the split that holds the new token encodes it while its first tiles are
 * in flight, the other splits never wait for it.  (For codecs the staged
 * kernel does not take, see kvq_decode_attn, and for multi-wave launches on
 * paged caches, the append is its own small launch just before the decode,
 * which waits for it only before reading the new row; same results.)
 *   k_new, v_new  device fp16 [B][H_kv][head_dim], 16-byte aligned
 * Everything else as for kvq_decode_attn.  A ctx_len outside the range
 * above appends nothing (and is clipped and reported as there). */
int kvq_decode_step(const void* q, const void* k_new, const void* v_new,
                    const kvq_codec* kc, const kvq_codec* vc,
                    const int8_t* signs_k, const int8_t* signs_v,
                    const kvq_plane* K, const kvq_plane* V,
                    const int32_t* ctx_len, int32_t B, int32_t H_q,
                    int32_t H_kv, int64_t max_ctx, float softmax_scale,
                    int32_t num_splits, void* workspace, int64_t ws_bytes,
                    int32_t* err_word, void* out, int32_t out_dtype,
                    void* stream);

/* kvq_decode_step for a caller whose step inputs and output live in host
 * memory: on `stream`, copies in_host to in_dev, runs kvq_decode_step on
 * in_dev and out_dev, and copies out_dev to out_host.  With in_dev and
 * out_dev both NULL, the kernel reads the inputs from in_host and writes the
 * output to out_host directly (the transfers happen inside the launch, with
 * no separate copies); both must then be page-locked host memory the device
 * can address (cudaHostAlloc or cudaHostRegister), which is checked, and
 * 16-byte aligned.
 *   in_host   host [q | k_new | v_new], fp16: B*H_q*head_dim values of q,
 *             then B*H_kv*head_dim of k_new and of v_new (the layouts of
 *             kvq_decode_step), caller-owned; page-locked memory makes the
 *             copies asynchronous, pageable memory makes them synchronous
 *   in_dev    device buffer of the same size, 16-byte aligned, caller-owned
 *   out_host  host buffer for the output (B*H_q*head_dim values of the
 *             out_dtype of kvq_decode_step), caller-owned
 *   out_dev   device buffer of the same size, 16-byte aligned
 * The step's result is in out_host once the stream has passed the call.
 * Errors as for kvq_decode_step, plus KVQ_EINVAL for a NULL host buffer,
 * one device buffer without the other, or unmapped host memory without
 * device buffers, and KVQ_ECUDA when a copy cannot be issued. */
int kvq_decode_step_host(const void* in_host, void* in_dev, void* out_host, void* out_dev,
                         const kvq_codec* kc, const kvq_codec* vc,
                         const int8_t* signs_k, const int8_t* signs_v,
                         const kvq_plane* K, const kvq_plane* V,
                         const int32_t* ctx_len, int32_t B, int32_t H_q,
                         int32_t H_kv, int64_t max_ctx, float softmax_scale,
                         int32_t num_splits, void* workspace, int64_t ws_bytes,
                         int32_t* err_word, int32_t out_dtype, void* stream);

/* The paged forms: kvq_encode_kv, kvq_decode_attn and kvq_decode_step with
 * K and V in paged planes (see kvq_paged_plane).  Results are identical to
 * the contiguous forms on the same rows; arguments and errors as there
 * (tokens pos0 .. pos0+T-1 of every sequence must lie below its capacity). */
int kvq_encode_kv_paged(const kvq_codec* kc, const int8_t* signs_k, const void* k,
                        const kvq_paged_plane* K, const kvq_codec* vc,
                        const int8_t* signs_v, const void* v, const kvq_paged_plane* V,
                        int32_t B, int32_t H_kv, int32_t T, int64_t pos0,
                        int32_t* err_word, void* stream);
int kvq_decode_attn_paged(const void* q, const kvq_codec* kc, const kvq_codec* vc,
                          const int8_t* signs_k, const int8_t* signs_v,
                          const kvq_paged_plane* K, const kvq_paged_plane* V,
                          const int32_t* ctx_len, int32_t B, int32_t H_q,
                          int32_t H_kv, int64_t max_ctx, float softmax_scale,
                          int32_t num_splits, void* workspace, int64_t ws_bytes,
                          int32_t* err_word, void* out, int32_t out_dtype,
                          void* stream);
int kvq_decode_step_paged(const void* q, const void* k_new, const void* v_new,
                          const kvq_codec* kc, const kvq_codec* vc,
                          const int8_t* signs_k, const int8_t* signs_v,
                          const kvq_paged_plane* K, const kvq_paged_plane* V,
                          const int32_t* ctx_len, int32_t B, int32_t H_q,
                          int32_t H_kv, int64_t max_ctx, float softmax_scale,
                          int32_t num_splits, void* workspace, int64_t ws_bytes,
                          int32_t* err_word, void* out, int32_t out_dtype,
                          void* stream);

/* Size of the scratch array built into the library for
 * kvq_decode_attn_noalloc (4 MiB of device memory per GPU that loads it). */
#define KVQ_NOALLOC_SCRATCH_BYTES (4u << 20)

/* kvq_decode_attn without a workspace argument, for callers that cannot
 * allocate device memory: a serving loop whose device memory all belongs to
 * its own pooling allocator, a plain C program with no allocator, or code
 * that must not risk the synchronisation or out-of-memory failure of a fresh
 * cudaMalloc.  (The TurboAngle page has no counterpart: this is a library
 * convenience.)  Arguments and results are those of kvq_decode_attn; the
 * scratch comes from a KVQ_NOALLOC_SCRATCH_BYTES array compiled into the
 * library, which every GPU that loads the library holds until the process
 * exits.  A call whose kvq_decode_workspace_bytes() exceeds that size returns
 * KVQ_EINVAL before any launch (fewer splits reduce it).  The first call on a
 * device looks up the array's device address (with that device current):
 * make it before any stream capture.  Each call first clears the completion
 * counters with an asynchronous memset on `stream`, then runs the checks and
 * the launch of kvq_decode_attn: a call that those checks reject returns
 * KVQ_EINVAL with the memset already queued (harmless: every complete decode
 * leaves the counters at zero anyway).  The call allocates nothing.  All calls share the one array, so calls whose kernels overlap on
 * the GPU race on it and must be ordered by the caller. */
int kvq_decode_attn_noalloc(const void* q, const kvq_codec* kc,
                            const kvq_codec* vc, const int8_t* signs_k,
                            const int8_t* signs_v, const kvq_plane* K,
                            const kvq_plane* V, const int32_t* ctx_len,
                            int32_t B, int32_t H_q, int32_t H_kv,
                            int64_t max_ctx, float softmax_scale,
                            int32_t num_splits, int32_t* err_word, void* out,
                            int32_t out_dtype, void* stream);

/* Test controls for the failure-detection tests.  Failures are made on the
 * host, or by a device wait that gives up early; nothing here faults, traps
 * or hangs the GPU.  Process-wide settings, not meant for production use.
 *   KVQ_TEST_RESET          restores every default (value ignored)
 *   KVQ_TEST_FAIL_LAUNCHES  value n >= 0: the next n kernel launches of this
 *                           library are not made; each call that would have
 *                           made one returns KVQ_ECUDA (as a failed launch
 *                           does) with nothing queued on its stream
 *   KVQ_TEST_WAIT_LIMIT     value n >= 0: decode kernels launched from now on
 *                           give up a wait for a staged tile (or for a free
 *                           stage) after n tries (n = 0: at once, without
 *                           trying) and set KVQ_DEVERR_TIMEOUT in err_word; such
 *                           a CTA contributes nothing to the output.  Copies
 *                           already issued are still waited for, with the
 *                           default limit of 2^22 tries, before a CTA exits.
 *   KVQ_TEST_DEBUG_CHECKS   value 1 / 0: the KVQ_DEBUG checks on / off for
 *                           the rest of the process, whatever the environment
 *                           says (KVQ_TEST_RESET returns to the environment)
 * Returns KVQ_OK, or KVQ_EINVAL for an unknown key or a negative value. */
#define KVQ_TEST_RESET 0
#define KVQ_TEST_FAIL_LAUNCHES 1
#define KVQ_TEST_WAIT_LIMIT 2
#define KVQ_TEST_DEBUG_CHECKS 3
int kvq_test_control(int32_t key, int64_t value);

/* Message for the last non-OK status returned on the calling thread
 * (empty string if none).  The pointer stays valid until the next call on
 * the same thread. */
const char* kvq_last_error(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
int32_t kvq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
