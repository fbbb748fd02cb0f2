// Prologue of the ARCHead logit path (ARCHead Sec. 3, the bracket (H B_w^T) of the logit
// formula, and its core analogue H B_c^T):
//   * Hh = fp16(H 2^-e_n), zero-padded to Npad rows -- the B operand of the residual
//     contraction, each token scaled by its power of two (token_shift);
//   * t  = (H [Q8(B_c) | Q8(B_w)]^T) 2^-e_n, N x (r_c + r_r) FP32 -- the rank terms' left
//     products (for the tcgen05 path, split into FP16 pieces inside the MMA's B image);
//   * tsc[n] = 2^e_n, by which the epilogues multiply token n's logits.
#include "tc_common.cuh"

namespace archead {
namespace {

// Block-wide maximum of v (blockDim.x a multiple of 32, at most 1024); every thread gets it.
__device__ __forceinline__ float block_max(float v, float* red32) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();  // red32 may still be read from the previous use
  if (lane == 0) red32[warp] = v;
  __syncthreads();
  v = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v = fmaxf(v, red32[w]);
  return v;
}

// One block per token row (grid-stride over rows): the row's largest |h| gives its scale
// 2^-e_n, then each thread converts 8 consecutive BF16 values at a time.  Rows n >= N are
// written as zeros.  Non-finite entries set kErrRangeH.
__global__ void __launch_bounds__(256) convert_h_kernel(const uint16_t* __restrict__ H,
                                                        __half* __restrict__ Hh,
                                                        float* __restrict__ tsc, int64_t N,
                                                        int64_t Npad, int64_t D,
                                                        unsigned* err) {
  __shared__ float red32[8];
  const int64_t chunks = D / 8;
  bool bad = false;
  for (int64_t n = blockIdx.x; n < Npad; n += gridDim.x) {
    float m = 0.f;
    if (n < N)
      for (int64_t c = threadIdx.x; c < chunks; c += blockDim.x)
        m = fmaxf(m, bf16x8_absmax(__ldg(reinterpret_cast<const uint4*>(H + n * D + c * 8))));
    const int e = token_shift(block_max(m, red32));
    const float sc = ldexpf(1.f, -e);
    if (n < N && threadIdx.x == 0) tsc[n] = ldexpf(1.f, e);
    for (int64_t c = threadIdx.x; c < chunks; c += blockDim.x) {
      uint4 out = make_uint4(0, 0, 0, 0);
      if (n < N) {
        const uint4 in = __ldg(reinterpret_cast<const uint4*>(H + n * D + c * 8));
        const uint32_t w[4] = {in.x, in.y, in.z, in.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float lo = __uint_as_float(w[k] << 16) * sc;
          const float hi = __uint_as_float(w[k] & 0xFFFF0000u) * sc;
          o[k] = h2_bits(__floats2half2_rn(lo, hi));
          // exponent field all ones: infinite or NaN
          bad |= ((o[k] & 0x7C00u) == 0x7C00u) | ((o[k] & 0x7C000000u) == 0x7C000000u);
        }
        out = make_uint4(o[0], o[1], o[2], o[3]);
      }
      *reinterpret_cast<uint4*>(Hh + n * D + c * 8) = out;
    }
  }
  if (bad) atomicOr(err, kErrRangeH);
}

// t[n, j] = 2^-e_n sum_d h[n, d] * fl32(B[j, d] * sB[j, d / g]) with j < r_c from B_c and
// the rest from B_w.  Block (token group of kTN, j); 256 threads stride over D, 8 columns
// each.  The block sees the whole rows of its tokens, so it finds each token's e_n itself
// (token_shift of the same row maximum as the conversion kernels).
constexpr int kTN = 8;

__global__ void __launch_bounds__(256) lowrank_t_kernel(
    const uint16_t* __restrict__ H, const int8_t* __restrict__ Bc,
    const float* __restrict__ sBc, const int8_t* __restrict__ Bw,
    const float* __restrict__ sBw, int r_c, int r_r, int64_t N, int64_t D, int g,
    float* __restrict__ t, __half* __restrict__ img, int nt, int64_t nkbt,
    unsigned* err) {
  allow_dependent_launch();
  const int j = blockIdx.y;
  const int RR = r_c + r_r;
  const int8_t* B;
  const float* sB;
  int jj;
  if (j < r_c) {
    B = Bc; sB = sBc; jj = j;
  } else {
    B = Bw; sB = sBw; jj = j - r_c;
  }
  const int64_t G = D / g;
  const int64_t n0 = (int64_t)blockIdx.x * kTN;
  const int nv = (N - n0) < kTN ? (int)(N - n0) : kTN;
  float acc[kTN], mx[kTN];
#pragma unroll
  for (int n = 0; n < kTN; ++n) acc[n] = mx[n] = 0.f;

  for (int64_t d0 = threadIdx.x * 8; d0 < D; d0 += 256 * 8) {
    uint2 braw = *reinterpret_cast<const uint2*>(B + jj * D + d0);
    const float s = sB[jj * G + d0 / g];
    float b[8];
    const int8_t* bq = reinterpret_cast<const int8_t*>(&braw);
#pragma unroll
    for (int k = 0; k < 8; ++k) b[k] = __fmul_rn((float)bq[k], s);
    // all kTN token rows are loaded (rows past N repeat the last one, and their sums are
    // never stored), so the loads carry no predicate and are in flight together
    uint4 hv[kTN];
#pragma unroll
    for (int n = 0; n < kTN; ++n)
      hv[n] = __ldg(reinterpret_cast<const uint4*>(H + (n0 + (n < nv ? n : nv - 1)) * D + d0));
#pragma unroll
    for (int n = 0; n < kTN; ++n) {
      mx[n] = fmaxf(mx[n], bf16x8_absmax(hv[n]));
      const uint32_t hw[4] = {hv[n].x, hv[n].y, hv[n].z, hv[n].w};
      float a = acc[n];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        a = fmaf(__uint_as_float(hw[k] << 16), b[2 * k], a);
        a = fmaf(__uint_as_float(hw[k] & 0xFFFF0000u), b[2 * k + 1], a);
      }
      acc[n] = a;
    }
  }
  // block reduction of the kTN sums and row maxima
  __shared__ float red[8][kTN], redm[8][kTN];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int n = 0; n < kTN; ++n) {
    float v = acc[n], m = mx[n];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      v += __shfl_xor_sync(0xffffffffu, v, o);
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    }
    if (lane == 0) {
      red[warp][n] = v;
      redm[warp][n] = m;
    }
  }
  __syncthreads();
  if (threadIdx.x < kTN && (int)threadIdx.x < nv) {
    float v = 0.f, m = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      v += red[w][threadIdx.x];
      m = fmaxf(m, redm[w][threadIdx.x]);
    }
    v *= ldexpf(1.f, -token_shift(m));  // exact: a power of two
    const int64_t n = n0 + threadIdx.x;
    // the image's rank blocks were zero-filled by the previous kernel (this one may be a
    // programmatic dependent launch of it)
    if (img) grid_dependency_wait();
    if (!img) {
      t[n * RR + j] = v;
    } else {
      // hi / lo FP16 pieces: t1 + t2 carries 22 significant bits of v
      const __half t1 = __float2half_rn(v);
      const __half t2 = __float2half_rn(v - __half2float(t1));
      if (!(fabsf(v) < 65504.f)) atomicOr(err, kErrRangeH);
      const uint32_t w = (uint32_t)__half_as_ushort(t1) | ((uint32_t)__half_as_ushort(t2) << 16);
      const int64_t tt = n / nt, nn = n - tt * nt;
      const int64_t kb = D / 128 + j / 32;
      *reinterpret_cast<uint2*>(img + tc_image_offset(tt, kb, nkbt, nt, nn, 4 * (j & 31))) =
          make_uint2(w, w);
    }
  }
}

}  // namespace

cudaError_t launch_prologue(const uint16_t* H, const archead_head* head, const Shapes& s,
                            int64_t Npad, __half* Hh, float* t, float* tsc, unsigned* err,
                            cudaStream_t st, int* launches) {
  {
    int64_t blocks = Npad < 148 * 16 ? Npad : 148 * 16;  // one block per row (grid-stride)
    if (blocks < 1) blocks = 1;
    convert_h_kernel<<<(unsigned)blocks, 256, 0, st>>>(H, Hh, tsc, s.N, Npad, s.D, err);
    ++*launches;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_lowrank_t(H, head, s, t, nullptr, 0, 0, err, st, launches);
}

cudaError_t launch_lowrank_t(const uint16_t* H, const archead_head* head, const Shapes& s,
                             float* t, __half* img, int nt, int64_t nkbt, unsigned* err,
                             cudaStream_t st, int* launches) {
  const int RR = s.r_c + s.r_r;
  if (RR > 0) {
    dim3 grid((unsigned)((s.N + kTN - 1) / kTN), RR);
    if (img) {  // tcgen05 path: may start while the image kernel still runs
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = grid;
      cfg.blockDim = dim3(256);
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      cudaError_t e = cudaLaunchKernelEx(&cfg, lowrank_t_kernel, H, head->Bc, head->sBc,
                                         head->Bw, head->sBw, s.r_c, s.r_r, s.N, s.D, s.g, t,
                                         img, nt, nkbt, err);
      if (e != cudaSuccess) return e;
    } else {
      lowrank_t_kernel<<<grid, 256, 0, st>>>(H, head->Bc, head->sBc, head->Bw, head->sBw,
                                             s.r_c, s.r_r, s.N, s.D, s.g, t, img, nt, nkbt,
                                             err);
    }
    ++*launches;
  }
  return cudaGetLastError();
}

}  // namespace archead
