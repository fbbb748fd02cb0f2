/*
 * archead.h -- C ABI of the ARCHead packed LM-head logit library (NVIDIA B200, sm_100a).
 *
 * The operation (ARCHead: Activation-Metric Residual Correction for Large Language Model
 * Output Heads, Sec. 3, the final approximation / logit formula and the inference
 * statement after Algorithm 1):
 *
 *     W_d = Q8(A_c) Q8(B_c) + SC4(R)          (INT8 low-rank core + packed INT4 residual)
 *     Y   = H W_d^T + (H B_w^T) A_w^T         (A_w row-wise INT8, B_w group-wise INT8)
 *
 * evaluated straight from packed storage; the dense V x D head never exists on the device.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor arguments are DEVICE pointers unless the name ends in _host; the caller
 *    owns every buffer it passes and the library never frees or retains them.
 *  - Row-major, densely packed.  BF16 and FP16 travel as uint16_t bit patterns.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  All work is enqueued
 *    on it and the calls return without synchronising, except archead_check and the
 *    _host variants.
 *  - Return value: ARCHEAD_OK (0) or a negative ARCHEAD_ERR_* code.  Argument errors are
 *    detected on the host before anything is enqueued.  Errors detected by a kernel
 *    (ARCHEAD_ERR_RANGE_H, ARCHEAD_ERR_TARGET) set a per-device error word; the affected
 *    outputs are non-finite; archead_check() reports and clears the word.
 *  - Temporary device memory (the N x (r_c + r_r) prologue product t, the FP16 image of H,
 *    the split-tile partials and counters, the NLL partials) is taken with
 *    cudaMallocAsync from a library-owned pool on `stream` and returned with
 *    cudaFreeAsync on the same stream.
 *  - Limits: g in {32, 64, 128, 256}; 128 <= D <= 2^20, D % 128 == 0 and D % g == 0;
 *    0 <= r_c, r_r <= 128; 1 <= V <= 8388480 (65535 blocks of 128 rows); 0 <= N < 2^31;
 *    N == 0 is a successful no-op.  V needs no multiple of any tile: the vocabulary tail
 *    is predicated.
 *  - Any finite BF16 H is accepted.  The kernels take FP16 operands, so each token row n
 *    is scaled by the power of two 2^-e_n, e_n = max(0, ilogb(max_d |h[n, d]|) - 14),
 *    which brings it below 2^15 exactly, and its logits are multiplied back by 2^e_n (a
 *    row with max |h| < 2^15 is not scaled).  Non-finite entries of H raise
 *    ARCHEAD_ERR_RANGE_H.  Where the rank terms run on the tensor cores (r_c and r_r
 *    multiples of 16 for N <= 16; every shape for N > 16) the scaled prologue products
 *    t 2^-e_n, t = H [Q8(B_c) | Q8(B_w)]^T, must stay below 65504 in magnitude, or the call
 *    raises ARCHEAD_ERR_RANGE_H.  Entries of the scaled rows below the FP16 normal range
 *    (2^-14; with one group code per 128 columns, g >= 128 and N <= 16, half of the
 *    columns are stored divided by 16) keep fewer bits, as rounding to FP16 does.
 */
#ifndef ARCHEAD_H_
#define ARCHEAD_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ARCHEAD_ABI_VERSION 2

enum archead_status {
  ARCHEAD_OK = 0,
  ARCHEAD_ERR_NULLPTR = -1,     /* a required pointer is NULL                         */
  ARCHEAD_ERR_ALIGN = -2,       /* a pointer is not 16-byte aligned                   */
  ARCHEAD_ERR_SHAPE = -3,       /* sizes disagree with the head or break a limit      */
  ARCHEAD_ERR_RANGE_H = -4,     /* H not finite, or a scaled rank product beyond FP16  */
  ARCHEAD_ERR_TARGET = -5,      /* a target id is outside [0, V)                      */
  ARCHEAD_ERR_TIMEOUT = -6,     /* a bounded device wait gave up                      */
  ARCHEAD_ERR_CUDA = -7,        /* a CUDA runtime call or launch failed               */
  ARCHEAD_ERR_UNSUPPORTED = -8, /* no kernel for this device / configuration          */
  ARCHEAD_ERR_NOMEM = -9        /* stream-ordered allocation failed                   */
};

/* Storage formats of a head (archead_head.format). */
enum archead_format {
  ARCHEAD_FMT_SC4 = 0, /* the ARCHead packed head below (default)                        */
  ARCHEAD_FMT_ROW8 = 1 /* Row INT8 baseline: W[v, d] = q8[v, d] * row_scale[v], no core,
                          no correction (the storage-matched comparison of Sec. 5)        */
};

/*
 * The packed head (the serialised module of Sec. 3: the SC4 residual and its scales, the
 * quantized core factors, the quantized correction factors and the shape metadata; no
 * dense head).  Every pointer is a device pointer, 16-byte aligned, owned by the caller.
 *
 *   r_nib   uint8  ceil(V/128)*128 x D/2  signed INT4 residual nibbles in the DEVICE
 *                           layout written by archead_repack_residual (see there)
 *   r_code  uint8  ceil(V/128)*128 x D/g  UINT8 code c of each residual group (g
 *                           columns), row-major; rows >= V are padding (any value)
 *   r_super bf16   V        per-row BF16 super-scale S; residual entry = q * c * S
 *   Ac int8 V x r_c, sAc f32 V         core left factor, one FP32 scale per row
 *   Bc int8 r_c x D, sBc f32 r_c x D/g core right factor, one FP32 scale per g columns
 *   Aw int8 V x r_r, sAw f32 V         correction left factor, row-wise
 *   Bw int8 r_r x D, sBw f32 r_r x D/g correction right factor, group-wise
 * A factor entry's value is the IEEE-single product of the INT8 value and its scale.
 * Factor pointers may be NULL when their rank is 0.
 *
 * format ARCHEAD_FMT_ROW8 (the Row INT8 baseline the paper compares with, about twice the
 * storage of the packed head):
 *   r_nib     int8 V x D, row-major (no repack): q8[v, d] in [-127, 127]
 *   row_scale float V: W[v, d] = q8[v, d] * row_scale[v] (the product taken exactly)
 *   r_c = r_r = 0; r_code, r_super and the factor pointers are not read (may be NULL); g
 *   must still be one of the supported values.  Such heads run on the token-block warp-MMA
 *   kernel for every N.
 */
typedef struct archead_head {
  int64_t V, D;
  int32_t r_c, r_r, g;
  int32_t format; /* archead_format */
  const uint8_t* r_nib;
  const uint8_t* r_code;
  const uint16_t* r_super;
  const int8_t* Ac;
  const float* sAc;
  const int8_t* Bc;
  const float* sBc;
  const int8_t* Aw;
  const float* sAw;
  const int8_t* Bw;
  const float* sBw;
  const float* row_scale; /* ARCHEAD_FMT_ROW8 only */
} archead_head;

/*
 * archead_logits -- Y = H W_d^T + (H B_w^T) A_w^T   (ARCHead Sec. 3, logit formula).
 *   H  bf16 N x D (device), Y float N x V (device, fully overwritten).
 *   N, V, D, r_c, r_r, g must equal the head's metadata (ARCHEAD_ERR_SHAPE otherwise).
 *   N <= 16 runs the persistent decode kernel (warp MMAs; each packed byte read once per
 *   call), larger N the tcgen05 kernel (tensor-memory accumulators); shapes whose shared-
 *   memory plans do not fit take a token-block warp-MMA kernel.  The main kernel starts
 *   while the prologue still runs (programmatic dependent launch).  Asynchronous on
 *   `stream`.
 *   Precision: H is rounded to FP16 and products accumulate in FP32.  Residual operands:
 *   exact q*c*2^-k in FP16 (N > 16), or raw nibble reads with a per-block offset
 *   correction and the group code applied to the FP32 block sum (N <= 16, g >= 128),
 *   else exact q*c.  Low-rank terms: FP32 (r not a multiple of 16, N <= 16) or FP16
 *   hi/lo pieces of the factor entries and of t on the tensor cores (about 22 bits).
 */
int archead_logits(const uint16_t* H, const archead_head* head, float* Y, int64_t N,
                   int64_t V, int64_t D, int r_c, int r_r, int g, void* stream);

/*
 * archead_nll -- per-token negative log-likelihood in nats (cross-entropy of Sec. 5):
 *   nll[n] = logsumexp_v Y[n, v] - Y[n, targets[n]], without writing the N x V logits.
 *   targets int32 N (device), nll_out float N (device).  A target outside [0, V) sets
 *   ARCHEAD_ERR_TARGET in the device error word and makes that token's nll NaN.
 */
int archead_nll(const uint16_t* H, const archead_head* head, const int32_t* targets,
                float* nll_out, int64_t N, int64_t V, int64_t D, int r_c, int r_r, int g,
                void* stream);

/*
 * archead_agreement -- how closely the packed head's next-token distribution follows a
 *   dense reference head on the same hidden states: the agreement measures of Sec. 5
 *   (Table 8 and the paragraph on it: the dense top-1 token kept among the packed head's
 *   top k, and the KL divergence), computed in the epilogue of the logit kernel without
 *   writing the packed logits.
 *   Y_dense        float N x V (device): the reference logits, e.g. H W^T with the dense
 *                  BF16 head (the caller computes them).
 *   k              1..16.
 *   topk_out       int32 N x k (device): per token the ids of the k largest packed logits,
 *                  in decreasing order; equal logits are ordered by the smaller id first;
 *                  -1 where V < k.
 *   top1_dense_out int32 N (device): argmax_v Y_dense[n, v] (equal values: smaller id).
 *   kl_out         float N (device): KL(P_dense || P_packed) = sum_v p_d (log p_d - log p_p)
 *                  in nats, with p = softmax over the V logits; NaN where Y_dense holds a
 *                  non-finite value.
 *   lse_out        float N (device, may be NULL): log sum_v exp(Y_packed[n, v]).
 *   The top-k agreement of a token is top1_dense_out[n] in topk_out[n, :k'] for k' <= k.
 *   Runs on the token-block warp-MMA kernel for every N.  Scratch: N x ceil(V/128) x
 *   (6 + 2k) x 4 bytes from the library's pool.  Asynchronous on `stream`.
 */
int archead_agreement(const uint16_t* H, const archead_head* head, const float* Y_dense,
                      int k, int32_t* topk_out, int32_t* top1_dense_out, float* kl_out,
                      float* lse_out, int64_t N, int64_t V, int64_t D, int r_c, int r_r, int g,
                      void* stream);

/*
 * archead_nll_partials -- one vocabulary shard's share of archead_nll (cross-entropy of
 *   Sec. 5, evaluated vocabulary-parallel).  `head` holds rows [v_begin, v_begin + V) of a
 *   head with v_total rows (its V-indexed components sliced, B_c and B_w whole); targets
 *   are global ids in [0, v_total).  For every token it writes partials[n] = (m, s, y)
 *   (float N x 3, device): m = max_v Y[n, v] and s = sum_v exp(Y[n, v] - m) over the
 *   shard's rows, and y = Y[n, target] if the shard owns the target row, else 0.  The
 *   logits are not written.  Requires 0 <= v_begin, v_begin + V <= v_total < 2^31
 *   (ARCHEAD_ERR_SHAPE otherwise); a target outside [0, v_total) sets ARCHEAD_ERR_TARGET.
 *   Asynchronous on `stream`.
 */
int archead_nll_partials(const uint16_t* H, const archead_head* head, const int32_t* targets,
                         int64_t v_begin, int64_t v_total, float* partials, int64_t N,
                         int64_t V, int64_t D, int r_c, int r_r, int g, void* stream);

/*
 * archead_nll_merge -- nll[n] from G shards' partials (float G x N x 3, device, as
 *   archead_nll_partials writes them, shard k at [k]): M = max_k m_k,
 *   nll = M + log(sum_k s_k exp(m_k - M)) - sum_k y_k, combined in shard order.  Together
 *   with an all-gather of the partials between the GPUs that hold the shards this equals
 *   archead_nll on the whole head (up to rounding).  1 <= G <= 65536.  Asynchronous on
 *   `stream`.
 */
int archead_nll_merge(const float* partials, int G, int64_t N, float* nll_out, void* stream);

/*
 * archead_logits_host -- archead_logits with HOST buffers: copies H_host (bf16 N x D) to
 * the device, evaluates, copies Y back into Y_host (float N x V), and synchronises
 * `stream` before returning.  Pinned host memory gives asynchronous copies.  The device
 * staging buffers come from the library's stream-ordered pool.
 *   When Y holds at least about 6 MB, the vocabulary is evaluated in chunks (at most 8,
 * each a multiple of 128 rows, about 3 MB of Y) and each chunk's logits are copied to
 * Y_host on a library-owned second stream while the next chunks run, so the host copy,
 * which takes longer than the kernels for all but the smallest N, overlaps them.  Each
 * chunk is an ordinary archead_logits call on a view of the head's rows; the chunks' FP32
 * sums may round differently from one call over the whole head (within 1e-4 max|Y|).
 * archead_last_launches() then counts the launches of all chunks.
 */
int archead_logits_host(const uint16_t* H_host, const archead_head* head, float* Y_host,
                        int64_t N, int64_t V, int64_t D, int r_c, int r_r, int g,
                        void* stream);

/* archead_nll_host -- archead_nll with host H, targets and nll buffers (synchronous). */
int archead_nll_host(const uint16_t* H_host, const archead_head* head,
                     const int32_t* targets_host, float* nll_host, int64_t N, int64_t V,
                     int64_t D, int r_c, int r_r, int g, void* stream);

/*
 * archead_repack_residual -- canonical residual nibbles -> device layout (load-time step).
 *   canon: uint8 V x D/2, byte b of a row holds column 2b in bits 0-3 and column 2b+1 in
 *          bits 4-7 (two's-complement INT4).
 *   dev:   uint8 Vpad x D/2 with Vpad = ceil(V/128)*128 (rows >= V are written as zeros),
 *          the same nibbles tiled for sequential streaming: the 128-column block kb of the
 *          128-row tile T is the contiguous 8 KB region starting at (T*(D/128) + kb)*8192;
 *          in it, the 16-byte chunk i (0..3) of tile row s starts at (i*128 + s)*16.  Chunk
 *          i of a row's block holds four 32-bit words, word w for the 8 columns
 *          32*w + 8*i + {0..7}; inside a word, nibble position p (bits 4p..4p+3) holds
 *          column 2p for p < 4 and column 2(p-4)+1 for p >= 4.
 *   canon and dev must not overlap.  D % 128 == 0.  Asynchronous on `stream`.
 */
int archead_repack_residual(const uint8_t* canon, uint8_t* dev, int64_t V, int64_t D,
                            void* stream);

/*
 * archead_dequant -- test and inspection hook: writes dequantised components as FP32.
 *   R_out  float nrows x D : SC4 residual rows [row0, row0 + nrows): q * c * S (exact)
 *   Ac_out float nrows x r_c, Aw_out float nrows x r_r : row-wise INT8 factors
 *   Bc_out float r_c x D, Bw_out float r_r x D : group-wise INT8 factors
 * Each INT8 entry is the single round-to-nearest-even product of value and scale.  Any
 * output may be NULL to skip it.  Reads the residual in the device layout.  A Row INT8
 * head (ARCHEAD_FMT_ROW8) gives ARCHEAD_ERR_UNSUPPORTED.
 */
int archead_dequant(const archead_head* head, int64_t row0, int64_t nrows, float* R_out,
                    float* Ac_out, float* Aw_out, float* Bc_out, float* Bw_out,
                    void* stream);

/*
 * archead_check -- synchronises `stream`, then reads and clears this device's error
 * word.  Returns ARCHEAD_OK, ARCHEAD_ERR_RANGE_H, ARCHEAD_ERR_TARGET, ARCHEAD_ERR_TIMEOUT
 * or ARCHEAD_ERR_CUDA (a pending CUDA error).
 */
int archead_check(void* stream);

/*
 * archead_test_hooks -- failure-detection hook of the test build (libarchead_testhooks.so,
 *   compiled with ARCHEAD_TEST_HOOKS); the product library returns ARCHEAD_ERR_UNSUPPORTED
 *   and changes nothing.  In the test build it sets, for later calls on this process, the
 *   bound of the decode kernel's (N <= 16) bounded mbarrier waits in SM cycles (default
 *   2^31) and the CTA index whose first consumer warp waits on a barrier that no thread
 *   ever arrives on (-1: none).  That wait gives up after the bound, the kernel finishes
 *   with ARCHEAD_ERR_TIMEOUT in the device error word (archead_check reports it) and the
 *   logits of the call are undefined; the device stays usable.  wait_limit_cycles < 1
 *   gives ARCHEAD_ERR_SHAPE.
 */
int archead_test_hooks(long long wait_limit_cycles, int stall_cta);

/* Human-readable text of a status code (static string, never NULL). */
const char* archead_strerror(int status);

/* ARCHEAD_ABI_VERSION of the loaded library. */
int archead_abi_version(void);

/*
 * archead_last_launches -- number of kernels the library launched during the most recent
 * successful archead_logits / archead_nll call on this host thread (for launch counting).
 */
int archead_last_launches(void);

/*
 * archead_logits_noalloc -- archead_logits that allocates no device memory.
 *   The paper has no counterpart to this entry point: it exists for callers that cannot
 *   let a library allocate, such as serving engines that reserve nearly all GPU memory up
 *   front for their own pool and account for every byte, or decode loops that must not
 *   enter an allocator between kernels.
 *   Same arguments, layouts, results and error codes as archead_logits.  Its temporary
 *   buffers (the FP16 copy of H, Npad x D with Npad = N rounded up to 8, 16, 32 or a
 *   multiple of 64, plus the N x (r_c + r_r) FP32 rank products, each rounded up to 256
 *   bytes) live in one fixed 2 MiB device array that every GPU loading the library holds
 *   until the process exits; larger requests return ARCHEAD_ERR_SHAPE before anything is
 *   enqueued (e.g. D = 4096 allows N <= 192 with r_c + r_r = 64).
 *   The first call on a device looks up that array's device address (cudaGetSymbolAddress)
 *   with the device current; make that first call before any stream capture.  The address
 *   is kept for the life of the process: after cudaDeviceReset on a device, do not call
 *   this entry point (or any other of this library) on that device again.
 *   All calls share the one array: calls whose kernels overlap on the GPU (different
 *   streams, or several host threads) race on it and must be serialised by the caller.
 *   Each call writes every scratch byte before reading it, so no clearing is needed.
 */
int archead_logits_noalloc(const uint16_t* H, const archead_head* head, float* Y, int64_t N,
                           int64_t V, int64_t D, int r_c, int r_r, int g, void* stream);

/*
 * archead_profile -- measurement hook for timing the main contraction kernel alone.
 *   archead_profile(1) clears the record and, from then on, each archead_logits /
 *   archead_nll call on this process records a pair of CUDA events on its stream around
 *   its residual-contraction kernel (up to 16384 pairs; later launches are not recorded).
 *   archead_profile(0) stops recording.  archead_profile_read synchronises on the
 *   recorded events and returns the summed kernel milliseconds and the launch count.
 *   Both return ARCHEAD_OK or ARCHEAD_ERR_CUDA.  Not thread-safe across devices.
 */
int archead_profile(int enable);
int archead_profile_read(double* total_ms, int* count);

#ifdef __cplusplus
}
#endif

#endif /* ARCHEAD_H_ */
