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
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
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

// Prologue: Hh = fp16(H) padded with zero rows to Npad, t = H [Q8(B_c) | Q8(B_w)]^T.
cudaError_t launch_prologue(const uint16_t* H, const archead_head* head, const Shapes& s,
                            int64_t Npad, __half* Hh, float* t, unsigned* err,
                            cudaStream_t st, int* launches);

// t = H [Q8(B_c) | Q8(B_w)]^T alone (N x (r_c + r_r) FP32).
cudaError_t launch_lowrank_t(const uint16_t* H, const archead_head* head, const Shapes& s,
                             float* t, cudaStream_t st, int* launches);

// tcgen05 path: token tile (16, 32, 64 or 128) for N tokens and r_c + r_r = RR; the
// blocked FP16 copy of H (Npad = N rounded up to the tile) and t; the contraction.
int tc_token_tile(int64_t N, int RR);
cudaError_t launch_prologue_blocked(const uint16_t* H, const archead_head* head,
                                    const Shapes& s, int nt, __half* Hb, float* t,
                                    unsigned* err, cudaStream_t st, int* launches);
cudaError_t launch_residual_tc(const __half* Hb, const float* t, const archead_head* head,
                               const Shapes& s, float* Y, unsigned* err, cudaStream_t st,
                               int* launches);

// Residual dequant-contraction over token blocks of up to 64 (mma.sync path).
// mode 0: write logits Y.  mode 1: write NLL partials (max, sum exp) per (token, vocabulary
// block) into part[N x residual_gemm_vblocks] and the target logit into tlogit[N].
cudaError_t launch_residual_gemm(const __half* Hh, const float* t, const archead_head* head,
                                 const Shapes& s, float* Y, const int32_t* targets,
                                 float2* part, float* tlogit, cudaStream_t st, int* launches,
                                 int mode);
int residual_gemm_vblocks(const Shapes& s);
int64_t residual_token_block(int64_t N);  // rows of the zero-padded FP16 copy of H

// nll[n] from the partials; a target outside [0, V) gives NaN and sets kErrTarget.
cudaError_t launch_nll_combine(const float2* part, const float* tlogit,
                               const int32_t* targets, const Shapes& s, float* nll,
                               unsigned* err, cudaStream_t st, int* launches);

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
