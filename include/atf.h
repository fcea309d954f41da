/*
 * atf.h -- C ABI of the B200 (sm_100a) library for causal GQA attention with
 * one distance window per RoPE frequency pair.
 *
 * Method: "ATFlash: RoPE-Frequenzen kuerzen Attention-Arbeit um bis zu 57
 * Prozent" (sudo-ai.de).  Section "Was ATFlash anders macht": RoPE rotates
 * each frequency pair of q and k; every pair gets its own distance window,
 * proportional to its wavelength, beyond which its query-key product is left
 * out, so far keys stay reachable through the slow pairs.  Section "Die Zahlen
 * - und ihre Grenze": prefill and decode kernels keep the online softmax
 * unchanged.  This library's reading of "proportional distance":
 *
 *   omega_i = theta^(-2i/d),  lambda_i = 2 pi / omega_i,  W_i = ceil(alpha * lambda_i)
 *   logit(m, n) = (1/sqrt d) * sum_{i : m - n <= W_i} (q~_{2i} k~_{2i} + q~_{2i+1} k~_{2i+1})
 *   (no active pair -> logit 0, kept in the softmax), then causal softmax and P.V.
 *   alpha = +infinity gives plain causal RoPE attention.
 *
 * Conventions (all entry points):
 *   - Tensors are dense, row-major, token-major: [batch][token][head][d] with d
 *     contiguous, unless stated otherwise.  Element type bf16 (ATF_BF16) or
 *     fp32 (ATF_FP32).  Device pointers must be 16-byte aligned.
 *   - RoPE pairs are interleaved: pair i = elements (2i, 2i+1); rotation by
 *     +p*omega_i counter-clockwise for a token at position p.
 *   - GQA: query head h uses key/value head h / (heads / kv_heads).
 *   - `stream` is a cudaStream_t (0 = legacy default stream).  Every call is
 *     asynchronous on it; the return value reports argument and launch errors
 *     only.  The caller owns every buffer; the library never frees caller
 *     memory.
 *   - Supported: d in {64, 128}; heads % kv_heads == 0; heads / kv_heads <= 8
 *     for decode; theta > 1; alpha > 0 (finite or +inf).
 *   - Errors: a non-zero atf_status; atf_last_error() gives the message of the
 *     last failing call on the calling thread.
 *   - The library looks up the device address of its error word once per device
 *     and keeps it for the process: do not call it again on a device after a
 *     cudaDeviceReset of that device.
 */
#ifndef ATF_H
#define ATF_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATF_OK = 0,
  ATF_ERR_INVALID_ARG = 1, /* null pointer, negative size, inconsistent shape */
  ATF_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. d = 96) */
  ATF_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  ATF_ERR_TIMEOUT = 4      /* a kernel's bounded wait expired (see atf_check) */
} atf_status;

typedef enum { ATF_BF16 = 0, ATF_FP32 = 1 } atf_dtype;

/* Which dimensions form RoPE frequency pair i (i < d/2): (2i, 2i+1) as in the
 * method's formula, or (i, i + d/2) as in rotate-half (NeoX-style) checkpoints
 * such as the Qwen2.5 family the pages measure on.  Pair i has the same
 * frequency theta^(-2i/d) and window W_i either way.  The attention kernels read
 * rotated queries and keys in the interleaved order; atf_rope_layout's
 * rotate-half modes write rotate-half pairs in that order. */
typedef enum { ATF_PAIRS_INTERLEAVED = 0, ATF_PAIRS_ROTATE_HALF = 1 } atf_pairing;

/* Window table.  Writes W_i = ceil(alpha * 2 pi / theta^(-2i/d)), i < d/2, into
 * the host array W_out (d/2 entries), evaluated in fp64.  alpha = +inf gives
 * INT64_MAX.  Host only; no GPU needed. */
atf_status atf_windows(int d, double theta, double alpha, long long* W_out);

/* RoPE + layout (the "RoPE rotates each frequency pair" step of "Was ATFlash
 * anders macht").
 *   x:         input  [batch][seq][heads][d], dtype.
 *   x_rot:     output [batch][seq][heads][d], dtype, may be NULL.  Token t is
 *              rotated at position pos_offset + t (angles in fp64).
 *   x_chunked: output [batch][heads][d/16][seq][16] (bf16 only), may be NULL:
 *              the pair-chunk-major key layout read by atf_decode (chunk c holds
 *              pairs 8c..8c+7 of every token contiguously).
 *   rotate:    0 = copy / re-layout only (for caches already rotated),
 *              1 = apply RoPE to interleaved pairs (2i, 2i+1),
 *              2 = apply RoPE to rotate-half pairs (i, i + d/2) and write pair i
 *                  to dims (2i, 2i+1) of x_rot / x_chunked (the order the
 *                  attention kernels read; x and x_rot must not alias),
 *              3 = no rotation, only that reordering (rotate-half caches that
 *                  are already rotated).
 *              Other values: ATF_ERR_INVALID_ARG. */
atf_status atf_rope_layout(const void* x, void* x_rot, void* x_chunked, int batch, int seq, int heads, int d,
                           long long pos_offset, double theta, int rotate, int dtype, void* stream);

/* Prefill, full form. */
typedef struct {
  const void* q;   /* [batch][q_len][heads][d]; query t sits at position q_offset + t */
  const void* k;   /* [batch][kv_len][kv_heads][d]; key n sits at position n */
  const void* v;   /* [batch][kv_len][kv_heads][d] */
  void* out;       /* [batch][q_len][heads][d], same dtype as q */
  int batch, q_len, kv_len, heads, kv_heads, d;
  long long q_offset; /* absolute position of query row 0; kv_len >= q_offset + q_len */
  int dtype;          /* atf_dtype: ATF_BF16 -> tensor-core kernel, ATF_FP32 -> fp32 CUDA-core kernel */
  int rotated;        /* 1: q and k are already RoPE-rotated and in the kernels' interleaved
                         pair order (e.g. by atf_rope_layout); 0: rotated here */
  double theta, alpha;
  unsigned long long* skipped_pairs; /* device, may be NULL: += number of (query head, query,
                                        key, pair) quadruples outside their window */
  void* workspace;                   /* device scratch for the rotated q, k when rotated == 0 */
  size_t workspace_bytes;            /* >= atf_prefill_workspace_bytes(...) when rotated == 0 */
  int pairing;        /* atf_pairing of the unrotated q, k (used when rotated == 0) */
} atf_prefill_args;

/* Scratch bytes atf_prefill_ex needs for rotated copies of q and k (0 if rotated). */
size_t atf_prefill_workspace_bytes(int batch, int q_len, int kv_len, int heads, int kv_heads, int d, int dtype,
                                   int rotated);

/* Prefill (rows a1..a6 of the hot path: windows, RoPE, windowed QK, online
 * softmax, P.V, epilogue + skip counter).  With alpha = +inf the dense
 * specialisation of the same kernel runs (no window logic compiled in). */
atf_status atf_prefill_ex(const atf_prefill_args* args, void* stream);

/* Prefill, short form: batch 1, q_len = kv_len = seq, q_offset 0, bf16,
 * unrotated q and k.  Scratch for the rotated copies is taken stream-ordered
 * from the device's default memory pool (cudaMallocAsync / cudaFreeAsync on
 * `stream`); use atf_prefill_ex with a workspace to avoid that. */
atf_status atf_prefill(const void* q, const void* k, const void* v, void* out, int seq, int heads, int kv_heads,
                       int d, double theta, double alpha, void* stream);

/* Device scratch bytes atf_prefill_host needs: device copies of q, k, v, their
 * rotated forms (not when rotated) and the output. */
size_t atf_prefill_host_workspace_bytes(int batch, int q_len, int kv_len, int heads, int kv_heads, int d,
                                        int rotated);

/* Prefill from host memory: the same operation and result as atf_prefill_ex on
 * device copies of the inputs, with the host<->device copies overlapped with
 * each other and with the kernels.
 *   args->q, k, v, out: HOST memory, shapes as in atf_prefill_ex.  Page-locked
 *       memory (cudaHostAlloc / cudaHostRegister) lets the copies overlap;
 *       pageable memory gives the same result with the copies serialised.
 *   args->workspace: DEVICE scratch of atf_prefill_host_workspace_bytes(...)
 *       bytes, 16-byte aligned.
 *   args->dtype: ATF_BF16 only (else ATF_ERR_UNSUPPORTED).
 *   args->skipped_pairs: device pointer or NULL, as in atf_prefill_ex.
 *   chunk_rows: query rows per pipeline chunk (> 0), or 0 for q_len / 8
 *       rounded up to a multiple of 256.
 * Work order: k and v are uploaded whole, then the query rows chunk by chunk
 * from the last chunk to the first; each chunk is rotated and attended (as a
 * chunked prefill at offset q_offset + first row of the chunk, on `stream`) as
 * soon as it is on the device, and its output rows are downloaded while later
 * chunks run.  The copies run on two streams the library creates once per
 * device and host thread; before returning, the call makes `stream` wait for
 * both, so `out` holds the result once `stream` has reached that point
 * (synchronise `stream` before reading it).  The same workspace must not be in
 * use by another call that may run concurrently. */
atf_status atf_prefill_host(const atf_prefill_args* args, int chunk_rows, void* stream);

/* Decode: one new query per sequence against a rotated key cache.
 *   q:          [batch][heads][d] bf16, NOT rotated; rotated here at position kv_len[b]-1
 *               with the given atf_pairing.
 *   pairing:    atf_pairing of q (the cache is in the interleaved pair order either way).
 *   k_chunked:  [batch][kv_heads][d/16][n_cache][16] bf16, keys already rotated at
 *               their positions, pair-chunk-major (see atf_rope_layout).
 *   v:          [batch][n_cache][kv_heads][d] bf16.
 *   out:        [batch][heads][d] bf16.
 *   kv_len:     HOST array of batch lengths, 1 <= kv_len[b] <= n_cache; keys
 *               0..kv_len[b]-1 are live and the query sits at kv_len[b]-1
 *               (its own key included).
 *   workspace:  device scratch of >= atf_decode_workspace_bytes(...) bytes
 *               (split-softmax partials).
 *   skipped_pairs: device counter, may be NULL (+= skipped (head, key, pair)).
 * Only the key chunks whose highest pair window still reaches a key are read
 * from memory; every value row is read. */
atf_status atf_decode(const void* q, const void* k_chunked, const void* v, void* out, int batch,
                      const long long* kv_len, long long n_cache, int heads, int kv_heads, int d, double theta,
                      double alpha, int pairing, void* workspace, size_t workspace_bytes,
                      unsigned long long* skipped_pairs, void* stream);

/* Scratch bytes atf_decode needs for `batch` sequences of at most max_kv_len keys. */
size_t atf_decode_workspace_bytes(int batch, int heads, int kv_heads, long long max_kv_len, int d);

/* Decode over a key range, for a sequence whose cache is split across devices
 * (each holds a contiguous range of positions) or otherwise into pieces.
 * Sequence b's piece holds n_keys[b] rotated keys in slots 0 .. n_keys[b]-1, slot
 * j at position key_pos0[b] + j; its query sits at position q_pos[b] (>= the last
 * key's position) and is rotated there.  Windows and the causal order use those
 * positions, so the pieces of a sequence give, merged, exactly atf_decode's
 * softmax over all keys.
 *   q, k_chunked, v, n_cache, heads, kv_heads, d, theta, alpha, pairing,
 *   workspace, skipped_pairs: as in atf_decode (workspace sized with
 *   atf_decode_workspace_bytes for the largest n_keys).
 *   n_keys, key_pos0, q_pos: HOST arrays of batch entries; n_keys[b] may be 0 (an
 *   empty piece merges as nothing).  q_pos[b] - key_pos0[b] must be below 2^31
 *   (the kernels hold distances and windows in 32 bits); a larger distance is
 *   rejected with ATF_ERR_UNSUPPORTED before any work.
 *   partial: DEVICE fp32 [batch][heads][d + 2]: the piece's softmax numerator
 *   (relative to its maximum), its maximum logit (log2 units, -inf when empty)
 *   and its row sum: the form atf_decode_merge reads. */
atf_status atf_decode_partial(const void* q, const void* k_chunked, const void* v, float* partial, int batch,
                              const long long* n_keys, const long long* key_pos0, const long long* q_pos,
                              long long n_cache, int heads, int kv_heads, int d, double theta, double alpha,
                              int pairing, void* workspace, size_t workspace_bytes,
                              unsigned long long* skipped_pairs, void* stream);

/* Merges n_parts partials of atf_decode_partial, stored one after the other
 * ([n_parts][batch][heads][d + 2] fp32, device), into out [batch][heads][d] bf16
 * (log-sum-exp: each part's numerator and row sum are scaled by 2^(its max -
 * the overall max)).  Parts whose maximum is -inf contribute nothing. */
atf_status atf_decode_merge(const float* partials, int n_parts, int batch, int heads, int d, void* out,
                            void* stream);

/* Decode without any allocation: the same computation as atf_decode, but the
 * split-softmax partials live in a fixed 8 MiB device array inside the library
 * instead of a caller workspace.  The pages have no counterpart of this entry
 * point; it exists for callers that cannot allocate device memory on the decode
 * path -- a host application whose own memory manager owns all device memory and
 * forbids allocations behind its back, or a latency-critical serving loop where
 * an allocation may synchronise the device -- and so cannot hand over a workspace.
 *   - Arguments as atf_decode, minus the workspace.
 *   - Fails with ATF_ERR_UNSUPPORTED (no work done) when the call needs more than
 *     atf_decode_noalloc_scratch_bytes() of scratch, i.e. when
 *     atf_decode_workspace_bytes(batch, heads, kv_heads, max kv_len, d) is larger.
 *   - The array is held on every GPU that loads the library until the process
 *     exits.  The first call on a device looks up its device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make that
 *     first call before any stream capture.  It calls no cudaMalloc, cudaFree or
 *     other allocating routine.  The cached address belongs to the device's
 *     current context: it does not survive cudaDeviceReset (or any other
 *     destruction of that context), after which this entry point must not be
 *     called again in the same process.
 *   - All calls on a device share the array and it keeps the previous call's
 *     contents (every value read is written first in the same call).  Calls whose
 *     kernels overlap on the GPU (e.g. on unordered streams) race on it. */
atf_status atf_decode_noalloc(const void* q, const void* k_chunked, const void* v, void* out, int batch,
                              const long long* kv_len, long long n_cache, int heads, int kv_heads, int d,
                              double theta, double alpha, int pairing, unsigned long long* skipped_pairs,
                              void* stream);

/* Size in bytes of atf_decode_noalloc's fixed device scratch array. */
size_t atf_decode_noalloc_scratch_bytes(void);

/* KV-cache append for a varlen batch: the step on either side of the decode
 * attention ("Was ATFlash anders macht": the decode side reads the rotated key
 * cache).  New tokens' keys are rotated at their positions and written into the
 * pair-chunk-major key cache atf_decode reads; their values are copied into the
 * token-major value cache.
 *   k_new, v_new:    [total_new][kv_heads][d] bf16: the new tokens of sequence 0,
 *                    then those of sequence 1, ... (total_new = sum of n_new).
 *   n_new:           HOST array, batch entries >= 0: new tokens of each sequence.
 *   pos:             HOST array, batch entries >= 0: position of sequence b's first
 *                    new token; its tokens take positions (and cache slots)
 *                    pos[b] .. pos[b] + n_new[b] - 1, with pos[b] + n_new[b] <= n_cache.
 *   k_cache_chunked: [batch][kv_heads][d/16][n_cache][16] bf16 (atf_rope_layout's
 *                    chunk-major layout, pairs in the interleaved order).
 *   v_cache:         [batch][n_cache][kv_heads][d] bf16.
 *   pairing:         atf_pairing of k_new.
 * Only the appended slots are written.  Rotation in fp64, one rounding to bf16
 * (the same values atf_rope_layout produces for those positions). */
atf_status atf_kv_append(const void* k_new, const void* v_new, void* k_cache_chunked, void* v_cache, int batch,
                         const int* n_new, const long long* pos, long long n_cache, int kv_heads, int d,
                         double theta, int pairing, void* stream);

/* FASA-style decode (page "FASA", section "Das FASA-Framework arbeitet in zwei
 * Hauptphasen"): a token importance predictor scores every cached key on a given
 * set of dominant RoPE frequency pairs, each query head keeps its `budget`
 * best keys, and attention runs over those keys only.
 *   q_rot:     [batch][heads][d] bf16, ALREADY rotated at the query's position
 *              (e.g. by atf_rope_layout), pairs interleaved.
 *   k_chunked: [batch][kv_heads][d/16][n_cache][16] bf16 rotated key cache (the
 *              layout atf_decode reads); v: [batch][n_cache][kv_heads][d] bf16.
 *   kv_len:    HOST array, batch entries in [1, n_cache]: keys 0..kv_len[b]-1.
 *   pair_mask: bit i set = pair i (dims 2i, 2i+1) is dominant; non-empty, bits
 *              below d/2 only.  Only the 8-pair cache chunks holding a dominant
 *              pair are read for the scores.
 *   budget:    keys kept per query head, 1..4096 (all keys when kv_len <= budget).
 * Score of key n for query head h: the partial dot product of q and k over the
 * dims of the dominant pairs, summed in fp32 on the tensor cores -- for each
 * 8-pair cache chunk holding a dominant pair, in ascending order, the chunk's
 * 16 bf16 products (zero for its non-dominant pairs) are added to the running
 * sum in one mma.sync step, in a fixed arrangement, so a key's score has the
 * same bits in every kernel of the call; -0 counts as +0.  (Such a step's
 * rounding is not documented; the tests hold each score to within
 * 18 * 2^-23 * (number of dominant chunks) * sum_j |q_j k_j| of the exact one,
 * and to the exact one where every partial sum is exact, e.g. small integers.)
 * The kept keys are the `budget` highest scores, equal scores by lower index,
 * chosen via a threshold from one key in 32 (an exact pass over every key runs
 * if fewer than `budget` keys reach it).  Output:
 * out[b][h] = softmax over the kept keys of (1/sqrt d) q.k (all d dims), times
 * their values, bf16.
 *   selected:  device int32 [batch][heads][budget] or NULL: the kept key indices,
 *              ascending, -1 past min(kv_len, budget).
 *   scores:    device fp32 [batch][heads][n_cache] or NULL: the scores (entries
 *              n >= kv_len[b] are not written).
 *   workspace: device scratch of atf_fasa_workspace_bytes(...) bytes (the
 *              size assumes selected is NULL; less is needed when it is given).
 * Streams: with batch > 1 the work of each sequence runs on one of four
 * streams the library creates on the device's first such call (kept for the
 * process, so they do not survive cudaDeviceReset), forked from `stream` and
 * joined back to it with events: the call stays ordered on `stream` and can be
 * captured into a CUDA graph.
 * Errors: d not 64/128, more than 8 query heads per kv head, batch above 64,
 * budget outside [1, 4096] -> ATF_ERR_UNSUPPORTED; bad sizes, mask or kv_len,
 * small workspace, null or misaligned pointers -> ATF_ERR_INVALID_ARG. */
atf_status atf_fasa_decode(const void* q_rot, const void* k_chunked, const void* v, void* out, int batch,
                           const long long* kv_len, long long n_cache, int heads, int kv_heads, int d,
                           unsigned long long pair_mask, int budget, int* selected, float* scores,
                           void* workspace, size_t workspace_bytes, void* stream);
size_t atf_fasa_workspace_bytes(int batch, int heads, long long n_cache, int budget, int d);

/* Synchronises `stream` and reports ATF_ERR_TIMEOUT if any kernel of this
 * library on the current device gave up a bounded wait since the last
 * atf_check (the device error word is cleared), ATF_ERR_CUDA on a CUDA error. */
atf_status atf_check(void* stream);

/* Failure-detection self test: launches one CTA that waits on a barrier that
 * nothing ever completes, with a wait limit of `limit_cycles` SM clocks; the
 * kernel records the expiry in the device error word and returns.  A following
 * atf_check(stream) returns ATF_ERR_TIMEOUT.  No fault, trap or hang. */
atf_status atf_selftest_timeout(long long limit_cycles, void* stream);

/* Message of the last failing call on this thread ("" if none). */
const char* atf_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ATF_H */
