// Internal declarations shared by the ARCHead CUDA sources (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/archead.h"

namespace archead {

// Bits of the per-device error word (set by kernels with atomicOr, read by archead_check).
enum : unsigned {
  kErrRangeH = 1u,
  kErrTarget = 2u,
  kErrTimeout = 4u,
};

// ---------------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// LOP3 computing (a & b) ^ c.
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Dequantise one device-layout word (8 signed INT4 nibbles) into four half2 pairs of
// q * c, exact in FP16 (|q * c| <= 2040).
//
// Each nibble is moved to mantissa bits 6..9 of an FP16 whose exponent encodes 16.0
// (pattern 0x4C00, unit in the last place 1/64), so the half reads 16 + n.  Flipping the
// nibble's top bit first turns two's complement q into offset binary n = q + 8, so the
// half is 24 + q.  One fused multiply-add with (c, -24c) gives q * c: the product
// (24 + q) * c is exact before rounding, -24c has at most 11 significant bits, and the
// exact result is representable, so the single rounding is exact.
//
// Output pair i holds (column 2i, column 2i + 1) of the word's 8 columns, low half first,
// for the in-word order of the device layout (nibble p holds column 2p for p < 4 and
// column 2(p - 4) + 1 for p >= 4).
__device__ __forceinline__ void dequant_word(uint32_t w, __half2 c2, __half2 nc24,
                                             __half2 out[4]) {
  const uint32_t mask = 0x03C003C0u;   // mantissa bits 6..9 of both halves
  const uint32_t magic = 0x4E004E00u;  // 0x4C00 (16.0) with bit 9 set: flips the sign bit
  uint32_t p0 = and_xor(w << 6, mask, magic);
  uint32_t p1 = and_xor(w << 2, mask, magic);
  uint32_t p2 = and_xor(w >> 2, mask, magic);
  uint32_t p3 = and_xor(w >> 6, mask, magic);
  out[0] = __hfma2(*reinterpret_cast<__half2*>(&p0), c2, nc24);
  out[1] = __hfma2(*reinterpret_cast<__half2*>(&p1), c2, nc24);
  out[2] = __hfma2(*reinterpret_cast<__half2*>(&p2), c2, nc24);
  out[3] = __hfma2(*reinterpret_cast<__half2*>(&p3), c2, nc24);
}

// Device nibble layout, tiled: rows are padded to a multiple of 128 and every 128-row
// tile's 128-column block (64 bytes per row) is one contiguous 8 KB region, so each tile
// streams sequentially from HBM.  Inside the region, 16-byte chunk i (i = 0..3) of row s
// of the tile sits at (i * 128 + s) * 16.  Chunk i of a row block holds the 32-bit words of
// the 32-column windows w = 0..3 for the eight columns 32w + 8i + {0..7}, and inside a word
// nibble p holds column 2p (p < 4) or 2(p - 4) + 1 (p >= 4).
__device__ __forceinline__ int64_t nib_chunk_offset(int64_t v, int64_t kb, int64_t nkb, int i) {
  return (((v >> 7) * nkb + kb) << 13) + (((int64_t)i << 7) + (v & 127)) * 16;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}

// D = A * B + D, m16n8k16, FP16 operands, FP32 accumulators (legacy warp-level MMA).
__device__ __forceinline__ void mma_f16_16816(float d[4], const uint32_t a[4],
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
// 16-byte copy that reads src_bytes (0 or 16) from global memory and zero-fills the rest.
__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, uint32_t src_bytes) {
  uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// Token scaling.  H enters as BF16, whose range far exceeds FP16's; the kernels take FP16
// operands.  Token n is therefore scaled by 2^-e_n with e_n = max(0, ilogb(m_n) - 14),
// m_n = max_d |h[n, d]| (0 for a zero or non-finite m_n), so every entry of the scaled row
// is below 2^15 in magnitude; scaling by a power of two is exact.  The rank products t of
// the token are scaled the same way, the logits come out scaled by 2^-e_n, and each
// epilogue multiplies them by 2^e_n (tsc[n]).  Every kernel that needs e_n computes it from
// the same row maximum, so they agree bit for bit.
__device__ __forceinline__ int token_shift(float m) {
  if (!(m <= 3.402823466e38f) || m == 0.f) return 0;  // zero, infinite or NaN
  const int e = ilogbf(m) - 14;
  return e > 0 ? e : 0;
}

// The largest |h| of eight BF16 values (a 16-byte chunk of a row).
__device__ __forceinline__ float bf16x8_absmax(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    m = fmaxf(m, fabsf(__uint_as_float(w[k] << 16)));
    m = fmaxf(m, fabsf(__uint_as_float(w[k] & 0xFFFF0000u)));
  }
  return m;
}

__device__ __forceinline__ uint2 ldg_stream8(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];\n"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ---------------------------------------------------------------------------------
// Host-side launchers (defined in the .cu files)
// ---------------------------------------------------------------------------------

struct Shapes {
  int64_t N, V, D;
  int r_c, r_r, g;
};

// Prologue: Hh = fp16(H 2^-e_n) padded with zero rows to Npad, t = (H [Q8(B_c) |
// Q8(B_w)]^T) 2^-e_n, tsc[n] = 2^e_n (token scaling, see token_shift).
cudaError_t launch_prologue(const uint16_t* H, const archead_head* head, const Shapes& s,
                            int64_t Npad, __half* Hh, float* t, float* tsc, unsigned* err,
                            cudaStream_t st, int* launches);

// t = (H [Q8(B_c) | Q8(B_w)]^T) 2^-e_n (N x (r_c + r_r) FP32).  With img != nullptr the products
// go instead, split into FP16 pieces, into the rank blocks of the tcgen05 B image (token
// tile nt, nkbt blocks per tile); a piece outside the FP16 range sets kErrRangeH.
cudaError_t launch_lowrank_t(const uint16_t* H, const archead_head* head, const Shapes& s,
                             float* t, __half* img, int nt, int64_t nkbt, unsigned* err,
                             cudaStream_t st, int* launches);

// tcgen05 path.  The MMA's B operand is a blocked FP16 image of the tokens: per token tile
// of nt rows, nkb = D / 128 blocks of H followed by nrb = ceil((r_c + r_r) / 32) rank
// blocks, each nt x 128 FP16 (see tc_image_offset).  Rank block b holds, for the factor
// index j = 32 b + i (i < 32), columns 4i..4i+3 = (t1, t2, t1, t2), where t1 = fp16(t_j)
// and t2 = fp16(t_j - t1) split the FP32 left product t = H [Q8(B_c) | Q8(B_w)]^T.
struct TcPlan {
  int nt;   // token tile: 16, 32, 64 or 128 (0: the shape does not fit this kernel)
  int sb;   // stages of the shared-memory ring of B blocks
  int nrb;  // rank blocks after the nkb blocks of H
  int sp;   // stages of the shared-memory ring of packed blocks
};
TcPlan tc_plan(const Shapes& s, bool nll);
// FP16 element offset of (token nn of token tile tt, column kk < 128 of block kb) in the
// blocked image with nkbt blocks per token tile: two 64-column halves of nt rows x 128
// bytes, the 16-byte chunk c of row nn stored at chunk c ^ (nn % 8) (the K-major 128-byte
// swizzle the MMA's shared-memory descriptor names).
__host__ __device__ __forceinline__ int64_t tc_image_offset(int64_t tt, int64_t kb,
                                                            int64_t nkbt, int nt, int64_t nn,
                                                            int kk) {
  return (tt * nkbt + kb) * (int64_t)nt * 128 + (int64_t)(kk >> 6) * nt * 64 + nn * 64 +
         ((((kk >> 3) & 7) ^ (int)(nn & 7)) << 3) + (kk & 7);
}
// Blocked image of H (zero rows up to the token tile) and its rank blocks.
// counters: ceil(V/128) words zeroed here (the per-tile counters of a split launch, or
// the work counter of the dynamic item order), or nullptr.
cudaError_t launch_prologue_blocked(const uint16_t* H, const archead_head* head,
                                    const Shapes& s, const TcPlan& plan, __half* Hb, float* tsc,
                                    unsigned* counters, unsigned* err, cudaStream_t st,
                                    int* launches);
// Bytes of scratch for a launch whose single token tile is split evenly over the CTAs
// (0 when the shape has more than one token tile).
size_t tc_split_scratch_bytes(const Shapes& s, const TcPlan& plan);
// Y != nullptr: write logits.  Y == nullptr: fused NLL, writing (max, sum exp) partials
// into part[N x ceil(V/128)] and target logits into tlogit[N] (see launch_nll_combine).
// scratch / counters (tc_split_scratch_bytes, launch_prologue_blocked): the split of a
// single token tile over the CTAs; with several token tiles, counters[0] is the work
// counter from which the CTAs take their items in order (nullptr: a fixed round-robin).
cudaError_t launch_residual_tc(const __half* Hb, const float* tsc, const archead_head* head,
                               const Shapes& s, const TcPlan& plan, float* Y,
                               const int32_t* targets,
                               float2* part, float* tlogit, float* scratch, unsigned* counters,
                               unsigned* err, cudaStream_t st, int* launches);

// Decode path (N <= 16): persistent bulk-copy-fed warp-MMA kernel with H resident in
// shared memory.  nt8 = 0 when the shape does not fit (then the token-block kernel runs).
struct DecPlan {
  int nt8;   // 8-token MMA column tiles: 1 (N <= 8) or 2 (N <= 16)
  int sp;    // packed ring stages
  int grid;  // CTAs (one per SM)
};
DecPlan dec_plan(const Shapes& s, bool nll);
size_t dec_image_bytes(const Shapes& s, const DecPlan& pl);  // resident H image
size_t dec_partial_bytes(const DecPlan& pl);                 // split-tile partials
// H image (tokens scaled by 2^-e_n, with the offset corrections and the token scales 2^e_n
// after it) + zeroed per-tile counters (ceil(V/128) words), then t (N x RR FP32, unscaled:
// the decode kernel divides by 2^e_n when it stages t).
cudaError_t launch_dec_prologue(const uint16_t* H, const archead_head* head, const Shapes& s,
                                const DecPlan& pl, __half* img, float* t, unsigned* counters,
                                unsigned* err, cudaStream_t st, int* launches);
// Y != nullptr: logits; else fused-NLL partials as in launch_residual_gemm mode 1.
cudaError_t launch_residual_dec(const __half* img, const float* t, const archead_head* head,
                                const Shapes& s, const DecPlan& pl, float* Y,
                                const int32_t* targets, float2* part, float* tlogit,
                                float4* scratch, unsigned* counters, unsigned* err,
                                cudaStream_t st, int* launches);

#ifdef ARCHEAD_TEST_HOOKS
// Failure-detection test builds: the bound of the decode kernel's mbarrier waits (SM
// cycles) and the CTA whose consumer warp 0 waits on a barrier that never completes
// (-1: none).
void set_dec_test_hooks(long long wait_limit, int stall_cta);
#endif

// Residual dequant-contraction over token blocks of up to 64 (mma.sync path).
// mode 0: write logits Y.  mode 1: write NLL partials (max, sum exp) per (token, vocabulary
// block) into part[N x residual_gemm_vblocks] and the target logit into tlogit[N].
cudaError_t launch_residual_gemm(const __half* Hh, const float* t, const float* tsc,
                                 const archead_head* head,
                                 const Shapes& s, float* Y, const int32_t* targets,
                                 float2* part, float* tlogit, cudaStream_t st, int* launches,
                                 int mode);
int residual_gemm_vblocks(const Shapes& s);
// Agreement with a dense reference head (mode 2 of the warp-MMA kernel, then a merge):
// per token the ids of the topk largest packed logits, the dense argmax, KL(dense ||
// packed) and the packed log-sum-exp.  Scratch: astat N x nvblk x 6 floats, akval and akid
// N x nvblk x topk each (nvblk = residual_gemm_vblocks).
cudaError_t launch_agreement(const __half* Hh, const float* t, const float* tsc,
                             const archead_head* head,
                             const Shapes& s, const float* Yd, int topk, float* astat,
                             float* akval, int* akid, int32_t* topk_out, int32_t* top1_dense,
                             float* kl_out, float* lse_out, cudaStream_t st, int* launches);
int64_t residual_token_block(int64_t N);  // rows of the zero-padded FP16 copy of H

// nll[n] from the partials; a target outside [0, V) gives NaN and sets kErrTarget.
cudaError_t launch_nll_combine(const float2* part, const float* tlogit,
                               const int32_t* targets, const Shapes& s, float* nll,
                               unsigned* err, cudaStream_t st, int* launches);

// Vocabulary-parallel NLL (csrc/nll_shard.cu).  A shard holds rows [v_begin, v_begin + V)
// of a head with v_total rows.  prep: shard-local targets (t - v_begin, or -1 when another
// shard owns the row) into tloc[N] and zeroed target logits; targets outside [0, v_total)
// set kErrTarget.  partials: the shard's (max, sum exp, target logit) per token, out[N][3].
// merge: nll[n] from G shard triples [G][N][3], combined in shard order.
cudaError_t launch_nll_shard_prep(const int32_t* targets, int64_t N, int64_t v_begin,
                                  int64_t V, int64_t v_total, int32_t* tloc, float* tlogit,
                                  unsigned* err, cudaStream_t st, int* launches);
cudaError_t launch_nll_partials(const float2* part, const float* tlogit, const Shapes& s,
                                float* out, cudaStream_t st, int* launches);
cudaError_t launch_nll_merge(const float* partials, int G, int64_t N, float* nll,
                             cudaStream_t st);

cudaError_t launch_repack(const uint8_t* canon, uint8_t* dev, int64_t V, int64_t D,
                          cudaStream_t st);

// Host helpers defined in archead_api.cu.
int validate_head_args(const archead_head* head, int64_t N, int64_t V, int64_t D, int r_c,
                       int r_r, int g);
unsigned* error_word_address();
cudaError_t launch_dequant(const archead_head* head, int64_t row0, int64_t nrows,
                           float* R_out, float* Ac_out, float* Aw_out, float* Bc_out,
                           float* Bw_out, cudaStream_t st);

}  // namespace archead
