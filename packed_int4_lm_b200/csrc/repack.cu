// Load-time layout step and the dequantisation inspection hook.
//
// Device nibble layout (see archead_repack_residual in archead.h and nib_chunk_offset):
// rows padded to a multiple of 128; each 128-row tile's 128-column block is a contiguous
// 8 KB region of 16-byte chunks, chunk i of tile row s at (i * 128 + s) * 16.  Chunk i of a
// row block holds, for the four 32-column windows w, the word of columns 32w + 8i + {0..7};
// inside a word nibble p holds column 2p (p < 4) or 2(p - 4) + 1 (p >= 4).  So a warp-quad
// thread's 16-byte chunk feeds its m16n8k16 A fragments for all four windows, a thread that
// owns a whole row reads its four chunks conflict-free, and the nibble pairs (p, p + 4)
// land in the two halves of one FP16x2 register.
#include "archead_internal.cuh"

namespace archead {
namespace {

__device__ __forceinline__ int nibble_pos_of_column(int i8) {
  return (i8 & 1) ? 4 + (i8 >> 1) : (i8 >> 1);
}

// One thread per 16-byte device chunk (row v, block kb, chunk i): its four words are the
// windows w = 0..3 of columns 32w + 8i + {0..7}.  Padding rows (v >= V) are zeros.
__global__ void __launch_bounds__(256) repack_kernel(const uint8_t* __restrict__ canon,
                                                     uint8_t* __restrict__ dev, int64_t V,
                                                     int64_t D) {
  const int64_t nkb = D / 128;
  const int64_t Vpad = (V + 127) / 128 * 128;
  const int64_t total = Vpad * nkb * 4;
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < total;
       q += (int64_t)gridDim.x * blockDim.x) {
    const int64_t v = q / (nkb * 4);
    const int64_t rem = q - v * nkb * 4;
    const int64_t kb = rem >> 2;
    const int i = (int)(rem & 3);
    uint32_t out[4] = {0u, 0u, 0u, 0u};
    if (v < V) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int64_t col0 = kb * 128 + 32 * w + 8 * i;
        // canonical: 8 consecutive columns = 4 bytes starting at byte col0 / 2 (4-aligned)
        const uint32_t cw = *reinterpret_cast<const uint32_t*>(canon + v * (D / 2) + col0 / 2);
#pragma unroll
        for (int i8 = 0; i8 < 8; ++i8)
          out[w] |= ((cw >> (4 * i8)) & 0xFu) << (4 * nibble_pos_of_column(i8));
      }
    }
    *reinterpret_cast<uint4*>(dev + nib_chunk_offset(v, kb, nkb, i)) =
        make_uint4(out[0], out[1], out[2], out[3]);
  }
}

__device__ __forceinline__ int residual_q(const uint8_t* __restrict__ dev, int64_t v, int64_t d,
                                          int64_t nkb) {
  const int64_t kb = d >> 7;
  const int within = (int)(d & 127);
  const int w = within >> 5, i = (within & 31) >> 3, i8 = within & 7;
  const uint32_t word =
      reinterpret_cast<const uint32_t*>(dev + nib_chunk_offset(v, kb, nkb, i))[w];
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
    const int q = residual_q(nib, v, d, D / 128);
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
  repack_kernel<<<grid_for((V + 127) / 128 * 128 * (D / 32)), 256, 0, st>>>(canon, dev, V, D);
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
