/*
 * kvq.h -- C ABI of the NVFP4 attention cache for NVIDIA B200 (sm_100a).
 *
 * A 4-bit attention cache: post-RoPE keys get static per-channel smoothing
 * (divide channel c by sqrt(absmax_c) from calibration, position 0 excluded;
 * the same factor is folded into the queries), optionally a normalised
 * Hadamard-128 rotation on head_dim; keys and values are quantised to E2M1 in
 * 16-element blocks along head_dim, each block with an E4M3 scale (block
 * absmax mapped to 6) under an FP32 per-tensor scale; attention reads the
 * packed cache directly.
 *
 * Sources (cited by page title and section):
 *   [P1] "NVFP4 attention cache on W4A4 Qwen3-8B: static key smoothing is
 *        near-lossless, key rotations hurt" (rstation.ai) -- setup paragraph,
 *        results table, observations, "For scale" paragraph.
 *   [P3] "QServe SmoothAttention (4-bit KV cache with an accuracy-preserving
 *        correction)" -- Activation scheme and Kernels fields.
 *   [P4] "OSFP4: Joint Optimization of Diagonal Smoothing and Block Scales for
 *        NVFP4 Quantization" -- Problem bullet, sec. 1, sec. 3, sec. D.1.
 *   [P5] "QuaRot KV cache 4-bit (rotated KV, no retained outlier channels)".
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library allocates no memory and keeps no state between calls.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  Host-side validation happens before any
 *     launch: on failure the call returns KVQ_EINVAL or KVQ_EUNSUPPORTED and
 *     launches nothing.  A launch failure returns KVQ_ECUDA.
 *   - Data-dependent faults (a page id outside the pool, a slot outside the
 *     cache, a length beyond the page table) never trap: the kernel skips the
 *     offending unit and ORs a KVQ_DEV_* bit into `*dev_status`, an int32 in
 *     device memory that the caller zeroes and reads back.  dev_status may be
 *     NULL, in which case such faults are skipped silently.
 *   - head_dim must be 128, page_size 16, num_kv_heads <= 8 and the GQA
 *     group num_q_heads / num_kv_heads <= 4 (KVQ_EUNSUPPORTED otherwise).
 *   - dtype arguments take KVQ_F32 or KVQ_BF16.
 *
 * Cache layout (owned by the caller, `kvq_page_bytes` bytes per page and
 * layer).  The cache of one layer is an array of pages; a page holds
 * page_size = 16 tokens of every kv head, as Hkv consecutive 2304-byte tiles:
 *     bytes [   0, 1024)  key codes    16 tokens x 64 B
 *     bytes [1024, 1152)  key scales   16 tokens x 8 B  (token-major)
 *     bytes [1152, 2176)  value codes  16 tokens x 64 B
 *     bytes [2176, 2304)  value scales 8 blocks x 16 B  (block-major)
 * Code byte j of a token row holds element 2j in its low nibble and element
 * 2j+1 in its high nibble (E2M1: s e1 e0 m).  Key scale byte t*8+b and value
 * scale byte b*16+t are the E4M3 scales of elements 16b..16b+15 of token t.
 * Keys are stored in the transformed basis (smoothed, optionally rotated).
 * A cache slot is page * 16 + offset.
 *
 * Mixed cache (shape->k_format = KVQ_K_BF16; [P1] results table, row "NVFP4
 * V only": the keys stay in BF16, the values are NVFP4).  The tile of one kv
 * head is 5248 bytes:
 *     bytes [   0, 4096)  keys         16 tokens x 128 bf16, untransformed
 *     bytes [4096, 5120)  value codes  16 tokens x 64 B
 *     bytes [5120, 5248)  value scales 8 blocks x 16 B  (block-major)
 * The keys are neither smoothed nor rotated (use_hadamard must be 0), and
 * the key entries of kvq_calib are not read.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t kvq_status;
enum {
    KVQ_OK = 0,
    KVQ_EINVAL = 1,         /* bad argument: null pointer, size, alignment  */
    KVQ_ECUDA = 2,          /* a CUDA call or launch failed                 */
    KVQ_EUNSUPPORTED = 3,   /* head_dim != 128, page_size != 16, no sm_100  */
    KVQ_EWORKSPACE = 4      /* workspace smaller than *_workspace_bytes     */
};

/* bits ORed into *dev_status by the kernels */
enum {
    KVQ_DEV_BAD_PAGE = 1,   /* page-table entry outside [0, num_pages)      */
    KVQ_DEV_BAD_SLOT = 2,   /* slot_mapping entry beyond the cache          */
    KVQ_DEV_BAD_LEN = 4,    /* seq_len < 0, or beyond max_pages_per_seq*16  */
    KVQ_DEV_TIMEOUT = 8,    /* a bounded wait on a copy gave up             */
    KVQ_DEV_BAD_WORKSPACE = 16 /* the workspace's counter header was not    */
                               /* zero-filled (see kvq_decode_attention)    */
};

enum { KVQ_F32 = 0, KVQ_BF16 = 1 };

/* key storage of the cache (kvq_shape.k_format) */
enum { KVQ_K_NVFP4 = 0, KVQ_K_BF16 = 1 };

#define KVQ_HEAD_DIM 128
#define KVQ_PAGE_SIZE 16
#define KVQ_TILE_BYTES 2304        /* one kv head of one page (see layout above) */
#define KVQ_TILE_BYTES_BF16K 5248  /* the same with KVQ_K_BF16 keys             */

typedef struct {
    int32_t num_layers;     /* L                                           */
    int32_t num_q_heads;    /* Hq = G * Hkv with GQA group G in 1..4        */
    int32_t num_kv_heads;   /* Hkv, 1..8 (even when use_hadamard)           */
    int32_t head_dim;       /* must be 128                                  */
    int32_t page_size;      /* must be 16                                   */
    int32_t use_hadamard;   /* 1: keys rotated by normalised Hadamard-128   */
    int32_t k_format;       /* KVQ_K_NVFP4, or KVQ_K_BF16 (mixed cache)     */
    int32_t use_klt;        /* 1: keys rotated by a static per-head KLT     */
} kvq_shape;

/* Static calibration state, device arrays of fp32 written by
 * kvq_calibrate_smoothing and read by every other call. */
typedef struct {
    float* k_smooth;        /* [L][Hkv][128] s = sqrt(absmax) (1 if zero)   */
    float* k_inv_smooth;    /* [L][Hkv][128] 1 / s                          */
    float* k_gscale;        /* [L] FP32 tensor scale g_K of the keys        */
    float* v_gscale;        /* [L] FP32 tensor scale g_V of the values      */
    float* k_klt;           /* [L][Hkv][128][128] KLT bases U (U[c][i] =    */
                            /* component c of vector i); read only with     */
                            /* use_klt, may be NULL otherwise               */
} kvq_calib;

typedef struct {
    uint8_t* data;              /* base of layer 0, 16-byte aligned          */
    int64_t layer_stride_bytes; /* bytes from one layer's pages to the next  */
    int32_t num_pages;          /* pages per layer                           */
} kvq_cache;

/* Bytes of one page of one layer: num_kv_heads * 2304 (5248 with BF16
 * keys); 0 on a bad shape. */
size_t kvq_page_bytes(const kvq_shape* shape);

/* Text of a status code (static storage). */
const char* kvq_status_string(kvq_status status);

/* Library version string, e.g. "kvq 0.1 sm_100a". */
const char* kvq_version(void);

/*
 * kvq_calibrate_smoothing -- static SmoothAttention factors and tensor scales.
 *
 * [P1] results table, row "K: static per-channel smoothing, sqrt(absmax)
 * from 4 C4 windows, position 0 excluded", and observation 2 (calibrate
 * without the sink; this is QServe's SmoothAttention, [P3]).  The FP32 tensor
 * scales follow the "global calibration-based scale" used for online
 * quantisation in [P4] sec. 3, here one per (layer, K|V), fitted so the
 * tensor's absmax maps to 6 * 448.
 *
 *   k_calib, v_calib  [L][num_windows][window_len][Hkv][128] post-RoPE keys
 *                     and values of the calibration windows, dtype.
 *   exclude_pos0      1: position 0 of every window is left out of the key
 *                     absmax (it still counts for the tensor scales).
 *   out               device arrays to fill (see kvq_calib):
 *                       A[l,h,c] = max_{w, t >= exclude_pos0} |k|
 *                       s = sqrt(A), or 1 when A = 0;  inv = 1/s
 *                       g_K = max |T(k)| / 2688 over all calibration tokens,
 *                       T = smoothing (+ rotation); g_V = max |v| / 2688;
 *                       a zero maximum gives 1.
 * Errors: KVQ_EINVAL for null pointers or non-positive sizes.
 */
kvq_status kvq_calibrate_smoothing(const kvq_shape* shape, const void* k_calib, const void* v_calib,
                                   int32_t dtype, int32_t num_windows, int32_t window_len,
                                   int32_t exclude_pos0, const kvq_calib* out, void* stream);

/*
 * kvq_calibrate_native -- tensor scales for keys kept in their native basis.
 *
 * [P1] results table, row "NVFP4 K only, native basis": the keys are
 * quantised without smoothing.  Writes s = 1 and inv = 1 for every (layer,
 * head, channel) -- so the append, the query pre-transform and attention
 * run unchanged -- and the FP32 tensor scales of kvq_calibrate_smoothing
 * over the unsmoothed keys: g_K = max |T(k)| / 2688 with T the optional
 * rotation alone, g_V = max |v| / 2688, over every calibration token; a zero
 * maximum gives 1.  Arguments and errors as kvq_calibrate_smoothing, without
 * exclude_pos0 (there is no smoothing absmax to leave the sink out of).
 */
kvq_status kvq_calibrate_native(const kvq_shape* shape, const void* k_calib, const void* v_calib,
                                int32_t dtype, int32_t num_windows, int32_t window_len,
                                const kvq_calib* out, void* stream);

/*
 * kvq_calibrate_klt -- smoothing followed by a static per-head KLT.
 *
 * [P1] results table, rows "K: static per-head KLT" and "K: static KLT +
 * smoothing" (the best WT-val row).  The smoothing factors are those of
 * kvq_calibrate_smoothing.  For each (layer, kv head) the basis U is the
 * eigenbasis of C = sum y y^T over the smoothed calibration keys y = k * inv
 * (positions t >= exclude_pos0 of every window), ordered by decreasing
 * eigenvalue, each vector signed so that its largest-magnitude component is
 * positive (fp32 cyclic Jacobi, 12 sweeps).  The keys are then transformed
 * as y'_i = sum_c U[c][i] y_c, one fp32 fused multiply-add chain per output
 * over c = 0..127; g_K = max |y'| / 2688 over every calibration token
 * (position 0 included), g_V as kvq_calibrate_smoothing.  out->k_klt must be
 * a [L][Hkv][128][128] fp32 device array; shape->use_klt must be 1 and
 * use_hadamard 0.  Errors as kvq_calibrate_smoothing.
 */
kvq_status kvq_calibrate_klt(const kvq_shape* shape, const void* k_calib, const void* v_calib,
                             int32_t dtype, int32_t num_windows, int32_t window_len,
                             int32_t exclude_pos0, const kvq_calib* out, void* stream);

/*
 * kvq_quantize_append -- transform, quantise and scatter tokens into the cache.
 *
 * [P1] setup paragraph: NVFP4 on post-RoPE cached keys and values, 16-blocks
 * along head_dim.  [P4] Problem bullet and sec. 1: absmax-to-6 block scaling;
 * sec. D.1: E2M1 values, an E4M3 scale per 16 entries, an FP32 tensor scale.
 * Per 16-element block of y (y = T(k) for keys, y = v for values):
 *     a = max|y|;  sf = E4M3(a * (1/(6 g)));  d = sf * g;
 *     r = 1/d (0 if d = 0);  code_i = E2M1(y_i * r)
 * each step one fp32 round-to-nearest-even; E4M3 and E2M1 saturate.
 *
 *   layer0, nlayers   layers [layer0, layer0 + nlayers) are written.
 *   k, v              [nlayers][num_tokens][Hkv][128], dtype, post-RoPE.
 *   slot_mapping      [num_tokens] int64 cache slot of each token (the same
 *                     for every layer); a negative slot skips the token.
 *   num_tokens        may be 0 (nothing is launched).
 * With KVQ_K_BF16 keys only the values are quantised; the keys are stored
 * as bf16 (bf16 input copied, fp32 input rounded to nearest-even).
 * Errors: KVQ_EINVAL for bad pointers/sizes; slots >= num_pages*16 set
 * KVQ_DEV_BAD_SLOT and are skipped.
 */
kvq_status kvq_quantize_append(const kvq_shape* shape, const kvq_calib* calib, const kvq_cache* cache,
                               int32_t layer0, int32_t nlayers, const void* k, const void* v,
                               int32_t dtype, const int64_t* slot_mapping, int32_t num_tokens,
                               int32_t* dev_status, void* stream);

/* Workspace bytes kvq_decode_attention needs for these sizes (0: none). */
size_t kvq_decode_workspace_bytes(const kvq_shape* shape, int32_t nlayers, int32_t batch,
                                  int32_t max_pages_per_seq);

/*
 * kvq_decode_attention -- one decode step of ragged GQA attention over the
 * packed cache, for every layer in [layer0, layer0 + nlayers) in one launch.
 *
 * The query carries the smoothing (and rotation) of the keys: q~ = q * s
 * (then H q~ / sqrt(128) with the rotation), so q~ . T(k) = q . k
 * ([P1] observation 2; [P3] SmoothAttention).  Attention is made
 * memory-bound on the 4-bit cache, as QServe's fused kernels are ([P3]
 * Kernels field): split-K over the pages of each sequence, dequantisation in
 * registers, online softmax with scale 1/sqrt(128), P.V, and a log-sum-exp
 * merge of the splits (in the same launch: the last split of each (layer,
 * sequence) to finish merges the partials of all of them, in split order).
 *
 *   q            [nlayers][batch][Hq][128], q_dtype, post-RoPE queries.
 *   page_table   [batch][max_pages_per_seq] int32 page ids (shared by all
 *                layers); entries past a sequence's length are not read.
 *   seq_lens     [batch] int32 cached tokens attended by each sequence
 *                (0 gives a zero output row).
 *   out          [nlayers][batch][Hq][128], out_dtype.
 *   workspace    >= kvq_decode_workspace_bytes(...) bytes, 16-byte aligned
 *                (may be NULL when that is 0).  Its first 4096 bytes are
 *                arrival counters of the split merge: they must hold zeros
 *                before the first call, and every call leaves them zero, so
 *                zero-fill a workspace once when allocating it (one buffer
 *                may then serve any sequence of decode and prefill calls).
 *                The rest is scratch (split partials, rotated queries) whose
 *                contents are undefined after the call.  A counter found
 *                at or above the split count (a header that was not
 *                zero-filled) sets KVQ_DEV_BAD_WORKSPACE; a smaller stale
 *                value cannot be told from an arrival and gives wrong rows.
 *                Calls that share a workspace must not overlap on the GPU.
 * With KVQ_K_BF16 keys the query is used as given (no smoothing, no
 * rotation, no key tensor scale): scores are q . k / sqrt(128).
 * Errors: KVQ_EINVAL / KVQ_EWORKSPACE on the host; KVQ_DEV_BAD_PAGE and
 * KVQ_DEV_BAD_LEN on the device (the affected rows are written as zeros),
 * KVQ_DEV_BAD_WORKSPACE (see workspace).
 */
kvq_status kvq_decode_attention(const kvq_shape* shape, const kvq_calib* calib, const kvq_cache* cache,
                                int32_t layer0, int32_t nlayers, const void* q, int32_t q_dtype,
                                const int32_t* page_table, int32_t max_pages_per_seq,
                                const int32_t* seq_lens, int32_t batch, void* out, int32_t out_dtype,
                                void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                void* stream);

/* Workspace bytes kvq_prefill_attention needs for these sizes (0: none;
 * only a KLT cache needs one).  The workspace follows the rules of
 * kvq_decode_attention's: its first 4096 bytes are left untouched. */
size_t kvq_prefill_workspace_bytes(const kvq_shape* shape, int32_t nlayers, int32_t batch,
                                   int32_t q_len);

/*
 * kvq_prefill_attention -- a chunk of q_len causal queries per sequence
 * against the packed cache (the chunk's own keys and values are appended
 * first with kvq_quantize_append).  Query i of sequence b sits at absolute
 * position q_start[b] + i and attends cached positions
 * j <= min(q_start[b] + i, seq_lens[b] - 1).  Same transform, scale and
 * output conventions as kvq_decode_attention.
 *
 *   q      [nlayers][batch][q_len][Hq][128], q_dtype.
 *   q_start [batch] int32.   out [nlayers][batch][q_len][Hq][128].
 * With a KVQ_K_BF16 cache the query is used as given (as in decode) and Q.K
 * runs on bf16 operands.
 */
kvq_status kvq_prefill_attention(const kvq_shape* shape, const kvq_calib* calib, const kvq_cache* cache,
                                 int32_t layer0, int32_t nlayers, const void* q, int32_t q_dtype,
                                 int32_t q_len, const int32_t* q_start, const int32_t* page_table,
                                 int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                                 void* out, int32_t out_dtype, void* workspace, size_t workspace_bytes,
                                 int32_t* dev_status, void* stream);

/*
 * kvq_prefill_attention_fp4 -- kvq_prefill_attention with Q.K taken on the
 * block-scaled FP4 tensor cores ("NVFP4 attention cache on W4A4 Qwen3-8B"
 * (rstation.ai), setup: W4A4, activations in NVFP4; "OSFP4" (paperlayer.ai
 * summary), Problem bullet, sec. 1 and sec. D.1).  The packed keys are the
 * MMA's operand as stored (E2M1 codes with their E4M3 block scales); the
 * query, after the same smoothing / rotation / KLT as kvq_prefill_attention,
 * is quantised to NVFP4 per row: g_q = amax(row) / 2688 (1 for a zero row),
 * then per 16-block sf = E4M3(absmax * (1 / (6 g_q))), d = val(sf) * g_q,
 * codes E2M1(x / d) -- the cache's quantiser with the row's own FP32 scale,
 * each step one IEEE fp32 rounding.  Scores are then
 * (sum over blocks of sf_q sf_k (codes . codes)) * g_q * g_K / sqrt(128);
 * softmax and P.V are those of kvq_prefill_attention.
 *
 * The result differs from kvq_prefill_attention's by the query's
 * quantisation error (4-bit codes), which is far above the fp32 rounding of
 * the unquantised query: compare it with attention on the dequantised query.
 * Same arguments, workspace, results and errors as kvq_prefill_attention;
 * a KVQ_K_BF16 (mixed) cache has no FP4 keys and returns KVQ_EINVAL.
 */
kvq_status kvq_prefill_attention_fp4(const kvq_shape* shape, const kvq_calib* calib, const kvq_cache* cache,
                                     int32_t layer0, int32_t nlayers, const void* q, int32_t q_dtype,
                                     int32_t q_len, const int32_t* q_start, const int32_t* page_table,
                                     int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                                     void* out, int32_t out_dtype, void* workspace, size_t workspace_bytes,
                                     int32_t* dev_status, void* stream);

/*
 * kvq_decode_attention_noalloc -- kvq_decode_attention without a workspace
 * argument, for callers that cannot allocate device memory (code running
 * inside a host runtime that owns the device-memory budget and forbids
 * stray allocations, or latency-critical paths that cannot afford
 * cudaMalloc's implicit device-wide synchronisation).  The pages have no
 * counterpart to this call; it exists only for such callers.
 *
 * Same arguments, results and errors as kvq_decode_attention, whose host
 * checks run first.  The split-K scratch is a static device array of
 * KVQ_NOALLOC_SCRATCH_BYTES inside the library, reserved on every GPU that
 * loads it until the process exits; the call allocates nothing.  A problem
 * whose kvq_decode_workspace_bytes exceeds that size returns KVQ_EWORKSPACE
 * (after the argument checks) and launches nothing.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and keeps it for that device's context; make that
 *     first call before any stream capture.  After a cudaDeviceReset the
 *     next call looks the address up again: make it outside a capture too.
 *   - The array is shared by all calls on a device and keeps the last
 *     call's contents.  It starts zero-filled (a static device array), which
 *     is what the split merge's counters at its start need, and each call
 *     leaves those counters zero again; the decode writes every partial
 *     before reading it.  Calls whose GPU work overlaps (other streams,
 *     other host threads) race on the array: serialise them.
 */
#define KVQ_NOALLOC_SCRATCH_BYTES (16u << 20)

kvq_status kvq_decode_attention_noalloc(const kvq_shape* shape, const kvq_calib* calib, const kvq_cache* cache,
                                        int32_t layer0, int32_t nlayers, const void* q, int32_t q_dtype,
                                        const int32_t* page_table, int32_t max_pages_per_seq,
                                        const int32_t* seq_lens, int32_t batch, void* out, int32_t out_dtype,
                                        int32_t* dev_status, void* stream);

/*
 * Elementwise format conversions with the kernels' own rounding routines,
 * for checking them against a reference: kvq_round_e2m1 goes through the
 * E2M1 routine every quantiser uses (the append, the KLT key append and the
 * FP4 query of kvq_prefill_attention_fp4), eight values per call with even
 * positions in its low-nibble operand and odd ones in its high-nibble
 * operand; kvq_round_e4m3 through the E4M3 routine of the block scales.
 * x: [n] fp32 device array; codes: [n] bytes, one code per byte (E2M1 in the
 * low nibble; E4M3 as a byte).  Round-to-nearest-even, saturating, sign kept.
 */
kvq_status kvq_round_e2m1(const float* x, uint8_t* codes, int64_t n, void* stream);
kvq_status kvq_round_e4m3(const float* x, uint8_t* codes, int64_t n, void* stream);

/*
 * kvq_selftest_wait_timeout -- failure-detection self-test.  Launches one
 * small kernel that runs the library's bounded shared-memory-barrier wait
 * (the one every copy hand-off in the attention and append kernels uses) on
 * a barrier nothing ever arrives at.  The wait gives up after limit_ns
 * nanoseconds (1 us .. 10 s) and ORs KVQ_DEV_TIMEOUT into *dev_status; no
 * fault is raised and the context stays usable.
 * Errors: KVQ_EINVAL for a null status or a limit out of range.
 */
kvq_status kvq_selftest_wait_timeout(int32_t* dev_status, int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
