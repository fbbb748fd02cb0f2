// Load-time layout step and the dequantisation inspection hook.
//
// Device nibble layout (see archead_repack_residual in archead.h): a row is cut into
// 128-column blocks of 16 32-bit words; word slot 4t + w of a block carries the columns
// 32w + 8t + {0..7}; inside the word, nibble p carries column 2p (p < 4) or
// 2(p - 4) + 1 (p >= 4).  One warp-quad 128-bit load then brings each thread the eight
// columns it dequantises into an m16n8k16 A fragment for each of four 32-column windows,
// and the nibble pairs (p, p + 4) land in the two halves of one FP16x2 register.
#include "archead_internal.cuh"

namespace archead {
namespace {

__device__ __forceinline__ int nibble_pos_of_column(int i8) {
  return (i8 & 1) ? 4 + (i8 >> 1) : (i8 >> 1);
}

__global__ void __launch_bounds__(256) repack_kernel(const uint8_t* __restrict__ canon,
                                                     uint8_t* __restrict__ dev, int64_t V,
                                                     int64_t D) {
  const int64_t words_per_row = D / 8;
  const int64_t total = V * words_per_row;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t v = i / words_per_row;
    const int64_t widx = i - v * words_per_row;  // device word index within the row
    const int64_t blk = widx >> 4;
    const int slot = (int)(widx & 15);
    const int t = slot >> 2, w = slot & 3;
    const int64_t col0 = blk * 128 + 32 * w + 8 * t;
    // canonical: 8 consecutive columns = 4 bytes starting at byte col0 / 2 (4-aligned)
    const uint32_t cw = *reinterpret_cast<const uint32_t*>(canon + v * (D / 2) + col0 / 2);
    uint32_t out = 0;
#pragma unroll
    for (int i8 = 0; i8 < 8; ++i8) {
      const uint32_t nib = (cw >> (4 * i8)) & 0xFu;
      out |= nib << (4 * nibble_pos_of_column(i8));
    }
    reinterpret_cast<uint32_t*>(dev + v * (D / 2))[widx] = out;
  }
}

__device__ __forceinline__ int residual_q(const uint8_t* __restrict__ dev_row, int64_t d) {
  const int64_t blk = d >> 7;
  const int within = (int)(d & 127);
  const int w = within >> 5, t = (within & 31) >> 3, i8 = within & 7;
  const uint32_t word =
      reinterpret_cast<const uint32_t*>(dev_row)[blk * 16 + 4 * t + w];
  const int nib = (int)((word >> (4 * nibble_pos_of_column(i8))) & 0xFu);
  return nib >= 8 ? nib - 16 : nib;
}

__global__ void __launch_bounds__(256) dequant_residual_kernel(
    const uint8_t* __restrict__ nib, const uint8_t* __restrict__ code,
    const uint16_t* __restrict__ sup, int64_t row0, int64_t nrows, int64_t D, int g,
    float* __restrict__ out) {
  const int64_t total = nrows * D;
  const int64_t G = D / g;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / D, d = i - r * D;
    const int64_t v = row0 + r;
    const int q = residual_q(nib + v * (D / 2), d);
    const float c = (float)code[v * G + d / g];
    const float S = bf16_bits_to_float(sup[v]);
    // q * c * S has at most 20 significant bits: exact in either order
    out[i] = __fmul_rn((float)q, __fmul_rn(c, S));
  }
}

__global__ void __launch_bounds__(256) dequant_rowwise_kernel(const int8_t* __restrict__ q,
                                                              const float* __restrict__ s,
                                                              int64_t row0, int64_t nrows,
                                                              int cols, float* __restrict__ out) {
  const int64_t total = nrows * cols;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / cols;
    const int64_t v = row0 + r;
    out[i] = __fmul_rn((float)q[v * cols + (i - r * cols)], s[v]);
  }
}

__global__ void __launch_bounds__(256) dequant_groupwise_kernel(const int8_t* __restrict__ q,
                                                                const float* __restrict__ s,
                                                                int rows, int64_t D, int g,
                                                                float* __restrict__ out) {
  const int64_t total = (int64_t)rows * D;
  const int64_t G = D / g;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = i / D, d = i - j * D;
    out[i] = __fmul_rn((float)q[i], s[j * G + d / g]);
  }
}

unsigned grid_for(int64_t n) {
  int64_t b = (n + 255) / 256;
  if (b > 148 * 32) b = 148 * 32;
  return (unsigned)(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_repack(const uint8_t* canon, uint8_t* dev, int64_t V, int64_t D,
                          cudaStream_t st) {
  repack_kernel<<<grid_for(V * D / 8), 256, 0, st>>>(canon, dev, V, D);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const archead_head* h, int64_t row0, int64_t nrows, float* R_out,
                           float* Ac_out, float* Aw_out, float* Bc_out, float* Bw_out,
                           cudaStream_t st) {
  if (R_out && nrows > 0)
    dequant_residual_kernel<<<grid_for(nrows * h->D), 256, 0, st>>>(
        h->r_nib, h->r_code, h->r_super, row0, nrows, h->D, h->g, R_out);
  if (Ac_out && nrows > 0 && h->r_c > 0)
    dequant_rowwise_kernel<<<grid_for(nrows * h->r_c), 256, 0, st>>>(h->Ac, h->sAc, row0,
                                                                     nrows, h->r_c, Ac_out);
  if (Aw_out && nrows > 0 && h->r_r > 0)
    dequant_rowwise_kernel<<<grid_for(nrows * h->r_r), 256, 0, st>>>(h->Aw, h->sAw, row0,
                                                                     nrows, h->r_r, Aw_out);
  if (Bc_out && h->r_c > 0)
    dequant_groupwise_kernel<<<grid_for((int64_t)h->r_c * h->D), 256, 0, st>>>(
        h->Bc, h->sBc, h->r_c, h->D, h->g, Bc_out);
  if (Bw_out && h->r_r > 0)
    dequant_groupwise_kernel<<<grid_for((int64_t)h->r_r * h->D), 256, 0, st>>>(
        h->Bw, h->sBw, h->r_r, h->D, h->g, Bw_out);
  return cudaGetLastError();
}

}  // namespace archead
