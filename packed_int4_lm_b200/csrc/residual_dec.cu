// Small-batch (decode) logits: the memory-bound regime of the ARCHead logit formula
//
//   Y[n, v] = S_v sum_d h[n, d] q[v, d] c[v, d / g]                 (SC4 residual, Sec. 3)
//           + sAc[v] sum_j Ac[v, j] t[n, j] + sAw[v] sum_j Aw[v, j] t[n, r_c + j]
//
// for N <= 16 tokens, where every packed byte is used by at most 16 tokens and the kernel
// has to stream the head at HBM speed.  Design:
//  * persistent grid, one CTA per SM: the last warp is a producer that bulk-copies (TMA
//    engine, no tensor map, no multicast) two-block stages of the 8 KB packed blocks of
//    128-row tiles into a shared-memory ring, plus each tile's group codes and INT8 factor
//    rows; for N <= 8 each consumer warp owns two 16-row groups of the tile (their H
//    fragments are loaded once for both) and three warps take the stages of the same rows
//    in turn, for N <= 16 each warp owns 16 rows and takes every stage; a warp iterates over
//    its own stages only and probes the next one's barrier one stage ahead;
//  * the FP16 hidden states of all (<= 16) tokens stay resident in shared memory for the
//    whole launch, stored with a chunk swizzle that makes the B-fragment reads
//    conflict-free;
//  * A fragments come from the ring with ldmatrix: in the tiled device layout the 16-byte
//    chunk i of 8 consecutive rows is 128 contiguous bytes, so each 8x8 matrix load is
//    conflict-free, and thread (g, q) receives word q of chunk i of row g -- exactly the
//    eight columns it feeds into an m16n8k16 fragment (raw magic-number nibble reads with
//    one group code per 128-column block, exact FP16 q*c otherwise);
//  * the work is split evenly over CTAs in units of (tile, 128-column block), so all CTAs
//    finish together.  A tile split between CTAs is finished by the CTA that arrives
//    last (an atomic counter per tile, no waiting): it sums the partial accumulators of
//    all contributors in CTA order, so the result does not depend on arrival order;
//  * epilogue: S_v times the accumulator plus the rank terms (mma.sync on the INT8 factor
//    rows and FP16 hi / lo pieces of t, or FP32 from t); MODE 1 writes split-vocabulary
//    (max, sum exp) partials and target logits instead of Y.
// Every mbarrier wait is bounded; a wait that gives up sets the device error word and the
// warp skips its remaining waits, so the launch always ends.
#include "tc_common.cuh"

namespace archead {
namespace {

constexpr int kDecRows = 8;  // 16-row groups of a 128-row tile (one warp each per stage)
constexpr int kDecPk = 8192;                            // packed block of one tile

struct DecParams {
  const __half* Himg;  // NTOK x D FP16, chunk-swizzled rows (dec_h_offset)
  const float* t;      // N x RR
  const uint8_t* nib;
  const uint8_t* code;  // Vpad x G
  const uint16_t* sup;
  const int8_t* Ac;
  const float* sAc;
  const int8_t* Aw;
  const float* sAw;
  float* Y;
  const int32_t* targets;
  float2* part;
  float* tlogit;
  float4* scratch;     // partial accumulators: [CTA][2 slots][256 threads][NT8]
  unsigned* counters;  // arrivals per tile (zeroed by the prologue)
  int64_t N, V, D;
  int r_c, r_r, g_shift;
  int sp;  // packed ring stages
  int64_t n_vtiles;
  unsigned* err;
  long long wait_limit;  // bound of every mbarrier wait, in SM cycles
  int stall_cta;         // test builds: the CTA whose consumer warp 0 waits on a dead barrier
};

// FP16 element offset of (token n, column d) in the resident H image: rows of D
// elements; the 16-byte chunk q = d / 8 is stored at q ^ 2 [bit 3 of q] ^ [n odd], which
// spreads the eight 16-byte reads of each quarter warp over distinct bank groups.
__host__ __device__ __forceinline__ int64_t dec_h_offset(int64_t n, int64_t d, int64_t D) {
  const int64_t q = d >> 3;
  const int64_t pq = q ^ (((q >> 3) & 1) << 1) ^ (n & 1);
  return n * D + pq * 8 + (d & 7);
}

template <int NT8>
struct DecCfg {
  static constexpr int NTOK = 8 * NT8;
  // consumer warps per set of rows, taking the ring stages in turn (latency hiding where
  // the registers allow it)
  static constexpr int PAR = NT8 == 1 ? 3 : 1;
  // 16-row groups per consumer warp: two for one token block (the H fragments are loaded
  // once for both, and a stage's handshake serves twice the work)
  static constexpr int RG = NT8 == 1 ? 2 : 1;
  static constexpr int WPP = kDecRows / RG;  // consumer warps per stage
  static constexpr int CONSUMERS = WPP * PAR;
  static constexpr int THREADS = (CONSUMERS + 1) * 32;  // + producer warp
};

__host__ __device__ inline size_t dec_round16(size_t x) { return (x + 15) & ~(size_t)15; }

struct DecSmem {
  size_t h, pk, codes, arow_c, arow_w, ts, ts16, red, xch, bars, total;
};

// Row stride in bytes of the FP16 t pieces: RR halves rounded up to 128 bytes plus 32, so
// the stride in 32-bit words is 8 mod 32 and the 64-bit B-fragment reads of a half warp
// (four tokens x four K offsets) fall in distinct banks.
__host__ __device__ inline size_t dec_ts16_stride(int RR) {
  return ((size_t)RR * 2 + 127) / 128 * 128 + 32;
}

// Shared-memory carve-up (offsets from a 128-byte aligned base).
template <int NT8, int MODE>
__host__ __device__ inline DecSmem dec_smem(int64_t D, int G, int r_c, int r_r, int sp) {
  constexpr int NTOK = DecCfg<NT8>::NTOK;
  DecSmem m;
  size_t o = 0;
  m.h = o;  // H image [NTOK x D] FP16, corr quads [D / 128][NTOK / 2] float4, scales [NTOK]
  o += dec_round16((size_t)NTOK * D * 2 + (size_t)(D / 128) * NTOK * 8 + (size_t)NTOK * 4);
  m.pk = o;  // ring of sp stages of two packed blocks
  o += (size_t)sp * 2 * kDecPk;
  m.codes = o;  // [2][128 x G]
  o += 2 * dec_round16((size_t)128 * G);
  m.arow_c = o;  // [2][128 x r_c]
  o += 2 * dec_round16((size_t)128 * r_c);
  m.arow_w = o;  // [2][128 x r_r]
  o += 2 * dec_round16((size_t)128 * r_r);
  m.ts = o;  // [NTOK][RR + 1] FP32
  o += dec_round16((size_t)NTOK * (r_c + r_r + 1) * 4);
  m.ts16 = o;  // [2 pieces][NTOK rows of dec_ts16_stride bytes] FP16 hi / lo of t
  o += (size_t)2 * NTOK * dec_ts16_stride(r_c + r_r);
  m.red = o;  // MODE 1: [8 warps][NTOK] float2
  o += MODE ? dec_round16((size_t)kDecRows * NTOK * 8) : 0;
  m.xch = o;  // [2][PAR - 1][256][NT8] float4 partial sums handed to the warps of parity 0
  o += (size_t)2 * (DecCfg<NT8>::PAR - 1) * 256 * NT8 * 16;
  m.bars = o;
  o += 256;
  m.total = o;
  return m;
}

// The CTA whose unit range holds unit u, for U units split over C CTAs as
// [U c / C, U (c + 1) / C).
__device__ __forceinline__ int64_t dec_cta_of(int64_t u, int64_t U, int64_t C) {
  return ((u + 1) * C + U - 1) / U - 1;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t saddr, uint32_t r[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr)
               : "memory");
}

// Bounded wait that is skipped once this warp has already given up.
__device__ __forceinline__ bool dec_wait(uint64_t* bar, uint32_t parity, unsigned* err,
                                         bool ok, long long limit) {
  if (!ok) return false;
  return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity, err, limit));
}

// Prologue of this path: the resident H image (zero rows up to NTOK), followed by the
// offset corrections, and zeroed tile counters.  The corrections of block kb are stored as
// quads (corr[kb][2i], corr[kb][2i + 1], corr[kb][2i], corr[kb][2i + 1]) for token pairs
// i: a quad is the C operand that starts an m16n8k16 chain of the decode kernel.  One warp per (token, block);
// lane l converts columns 4l .. 4l + 3 of the block.
//
// With scale_b (one group code per 128-column block), the kernel feeds the MMA the raw
// magic-number reads of the nibbles: 1032 + q for columns with (d & 2) == 0 and
// 1152 + 16 q for the others, whose H values are stored divided by 16 (exact: a power of
// two).  Each k-block sum then carries the constant 1032 sum_A b + 1152 sum_B b over the
// stored values b; corr holds its negation, from which the kernel's MMA chain of the block
// starts, so the chain ends at the block's dot product.
// Each token is scaled by 2^-e_n (token_shift of its row maximum, which every warp of the
// token finds from the whole row: 16 KB per warp at most, from L2), and tsc[n] = 2^e_n
// follows the corrections (1 for the zero rows).  Non-finite entries set kErrRangeH.
// Runs on blocks blk of nblk.
__device__ __forceinline__ void dec_convert_h(const uint16_t* __restrict__ H,
                                              __half* __restrict__ img, int64_t N, int ntok,
                                              int64_t D, int scale_b,
                                              unsigned* __restrict__ counters,
                                              int64_t n_counters, unsigned* err, int64_t blk,
                                              int64_t nblk) {
  const int64_t nkb = D / 128;
  const int lane = threadIdx.x & 31;
  const int64_t gw = (blk * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (nblk * (int64_t)blockDim.x) >> 5;
  float* corr = reinterpret_cast<float*>(img + (int64_t)ntok * D);  // [nkb][ntok / 2] quads
  float* tsc = corr + nkb * ntok * 2;                                 // [ntok]
  bool bad = false;
  for (int64_t wi = gw; wi < (int64_t)ntok * nkb; wi += nw) {
    const int64_t n = wi / nkb, kb = wi - n * nkb;
    const int64_t d = kb * 128 + 4 * lane;
    float f[4] = {0.f, 0.f, 0.f, 0.f};
    float sc = 1.f;
    if (n < N) {
      const uint2 in = *reinterpret_cast<const uint2*>(H + n * D + d);
      f[0] = __uint_as_float(in.x << 16);
      f[1] = __uint_as_float(in.x & 0xFFFF0000u);
      f[2] = __uint_as_float(in.y << 16);
      f[3] = __uint_as_float(in.y & 0xFFFF0000u);
      float m = 0.f;  // the row maximum, sixteen 16-byte loads in flight per lane at a time
      for (int64_t c0 = lane; c0 < D / 8; c0 += 16 * 32) {
        uint4 v[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          v[q] = c0 + 32 * q < D / 8 ? __ldg(reinterpret_cast<const uint4*>(H + n * D + (c0 + 32 * q) * 8))
                                     : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int q = 0; q < 16; ++q) m = fmaxf(m, bf16x8_absmax(v[q]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const int e = token_shift(m);
      sc = ldexpf(1.f, -e);
      if (kb == 0 && lane == 0) tsc[n] = ldexpf(1.f, e);
#pragma unroll
      for (int k = 0; k < 4; ++k) f[k] *= sc;  // exact: a power of two
    } else if (kb == 0 && lane == 0) {
      tsc[n] = 1.f;
    }
    float sum = 0.f;
    __half hv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool typeb = ((d + e) & 2) != 0;
      hv[e] = __float2half_rn(scale_b && typeb ? f[e] * 0.0625f : f[e]);
      const float b = __half2float(hv[e]);
      bad |= !(fabsf(b) <= 65504.f);  // only a non-finite h after the scaling
      sum += (typeb ? 1152.f : 1032.f) * b;
    }
    const uint32_t lo = (uint32_t)__half_as_ushort(hv[0]) | ((uint32_t)__half_as_ushort(hv[1]) << 16);
    const uint32_t hi = (uint32_t)__half_as_ushort(hv[2]) | ((uint32_t)__half_as_ushort(hv[3]) << 16);
    *reinterpret_cast<uint2*>(img + dec_h_offset(n, d, D)) = make_uint2(lo, hi);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
      const int64_t q = (kb * (ntok / 2) + (n >> 1)) * 4 + (n & 1);
      corr[q] = corr[q + 2] = scale_b ? -sum : 0.f;
    }
  }
  for (int64_t i = blk * (int64_t)blockDim.x + threadIdx.x; i < n_counters;
       i += nblk * (int64_t)blockDim.x)
    counters[i] = 0u;
  if (bad) atomicOr(err, kErrRangeH);
}

// t[n, j] = sum_d h[n, d] fl32(B[j, d] s[j, d / g]) for the N <= 16 tokens of this path,
// B = [Q8(B_c) | Q8(B_w)]: one block per factor index j, 256 threads striding over D, 8
// columns each.  All of an iteration's loads (the 8 factor bytes, their scale and the 8
// columns of every token) are issued before its FMAs, so an iteration costs one memory
// latency whatever N is.
constexpr int kDecPrologueThreads = 256;

__device__ __forceinline__ void dec_lowrank_t(const uint16_t* __restrict__ H,
                                              const int8_t* __restrict__ Bc,
                                              const float* __restrict__ sBc,
                                              const int8_t* __restrict__ Bw,
                                              const float* __restrict__ sBw, int r_c, int r_r,
                                              int64_t N, int64_t D, int g, float* __restrict__ t,
                                              int j) {
  const int RR = r_c + r_r;
  const int8_t* B = j < r_c ? Bc + (int64_t)j * D : Bw + (int64_t)(j - r_c) * D;
  const float* sB = j < r_c ? sBc + (int64_t)j * (D / g) : sBw + (int64_t)(j - r_c) * (D / g);
  float acc[16];
#pragma unroll
  for (int n = 0; n < 16; ++n) acc[n] = 0.f;
  for (int64_t d0 = threadIdx.x * 8; d0 < D; d0 += kDecPrologueThreads * 8) {
    const uint2 braw = *reinterpret_cast<const uint2*>(B + d0);
    const float sc = sB[d0 / g];
    // all 16 token rows are loaded (rows past N repeat the last one, and their sums are
    // never stored), so the loads carry no predicate and issue together
    uint4 hv[16];
#pragma unroll
    for (int n = 0; n < 16; ++n)
      hv[n] = __ldg(reinterpret_cast<const uint4*>(H + (n < N ? n : N - 1) * D + d0));
    const int8_t* bq = reinterpret_cast<const int8_t*>(&braw);
    float b[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) b[k] = __fmul_rn((float)bq[k], sc);
#pragma unroll
    for (int n = 0; n < 16; ++n) {
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
  __shared__ float red[kDecPrologueThreads / 32][16];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    float v = acc[n];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp][n] = v;
  }
  __syncthreads();
  if ((int64_t)threadIdx.x < N) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kDecPrologueThreads / 32; ++w) v += red[w][threadIdx.x];
    t[(int64_t)threadIdx.x * RR + j] = v;  // unscaled: the decode kernel applies 2^-e_n
  }
}

// The whole prologue of this path in one launch: blocks [0, nconv) build the H image, its
// corrections and the zeroed counters; the next r_c + r_r blocks form t.
__global__ void __launch_bounds__(kDecPrologueThreads) dec_prologue_kernel(
    const uint16_t* __restrict__ H, __half* __restrict__ img, int64_t N, int ntok, int64_t D,
    int scale_b, unsigned* __restrict__ counters, int64_t n_counters, int nconv,
    const int8_t* __restrict__ Bc, const float* __restrict__ sBc,
    const int8_t* __restrict__ Bw, const float* __restrict__ sBw, int r_c, int r_r, int g,
    float* __restrict__ t, unsigned* err) {
  allow_dependent_launch();  // the main kernel may start streaming the packed head
  if ((int)blockIdx.x < nconv)
    dec_convert_h(H, img, N, ntok, D, scale_b, counters, n_counters, err, blockIdx.x, nconv);
  else
    dec_lowrank_t(H, Bc, sBc, Bw, sBw, r_c, r_r, N, D, g, t, (int)blockIdx.x - nconv);
}

constexpr int kDecMaxSP = 8;

// Whether the producer copies the tile's INT8 factor rows into shared memory (each bulk
// copy must be a multiple of 16 bytes; a ragged last tile may read them from global).
__host__ __device__ __forceinline__ bool dec_arow_copy(int64_t rows, int r_c, int r_r) {
  return ((rows * r_c) % 16) == 0 && ((rows * r_r) % 16) == 0;
}

// Raw magic-number reads of the eight nibbles of a device-layout word (no FP16 math):
// pairs 0 and 2 read 1032 + q, pairs 1 and 3 read 1152 + 16 q (see dec_convert_h).
__device__ __forceinline__ void nibble_reads(uint32_t w, uint32_t x[4]) {
  const uint32_t w2 = w >> 8;
  x[0] = and_xor(w, 0x000F000Fu, 0x64086408u);
  x[1] = and_xor(w, 0x00F000F0u, 0x64806480u);
  x[2] = and_xor(w2, 0x000F000Fu, 0x64086408u);
  x[3] = and_xor(w2, 0x00F000F0u, 0x64806480u);
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}

// m16n8k16 FP16 MMA whose chain starts from the quad c (C operand).
__device__ __forceinline__ void mma_f16_16816_q(float d[4], const uint32_t a[4], uint32_t b0,
                                                uint32_t b1, uint4 c) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%10, %11, %12, %13};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(c.x), "r"(c.y),
        "r"(c.z), "r"(c.w));
}

// NB (1 or 2) consecutive blocks with one group code each (g >= 128) for RG 16-row groups:
// raw nibble reads (nibble_reads) times the resident B image (each B fragment loaded once
// for all row groups), one chain of eight MMAs per (row group, block) starting from the
// block's negated offset constant (a quad of corr), then acc += code * chain.  hs: shared
// address of this thread's H row (token gid) at block kb2, chunk 0; cq: shared address of
// its corr quad at block kb2.
template <int NT8, int NB, int RG>
__device__ __forceinline__ void dec_blocks_q(const uint32_t (&wlo)[RG][2][4],
                                             const uint32_t (&whi)[RG][2][4],
                                             const uint32_t (&clo)[RG][2],
                                             const uint32_t (&chi)[RG][2], uint32_t hs,
                                             uint32_t hj, const uint32_t (&hoff)[4],
                                             uint32_t cq, float (&acc)[RG][NT8][4]) {
  constexpr int NTOK = 8 * NT8;
  float t[RG][NB][NT8][4];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      uint32_t a0[RG][4], a1[RG][4];
#pragma unroll
      for (int r = 0; r < RG; ++r) {
        uint32_t xa[4], xb[4];
        nibble_reads(wlo[r][b][c], xa);
        nibble_reads(whi[r][b][c], xb);
        a0[r][0] = xa[0]; a0[r][1] = xb[0]; a0[r][2] = xa[1]; a0[r][3] = xb[1];
        a1[r][0] = xa[2]; a1[r][1] = xb[2]; a1[r][2] = xa[3]; a1[r][3] = xb[3];
      }
#pragma unroll
      for (int j = 0; j < NT8; ++j) {
        const uint4 hv = lds128(hs + j * hj + b * 256 + hoff[c]);
        uint4 cqv = make_uint4(0, 0, 0, 0);
        if (c == 0) cqv = lds128(cq + (b * (NTOK / 2) + 4 * j) * 16);
#pragma unroll
        for (int r = 0; r < RG; ++r) {
          if (c == 0)
            mma_f16_16816_q(t[r][b][j], a0[r], hv.x, hv.y, cqv);
          else
            mma_f16_16816(t[r][b][j], a0[r], hv.x, hv.y);
          mma_f16_16816(t[r][b][j], a1[r], hv.z, hv.w);
        }
      }
    }
#pragma unroll
  for (int r = 0; r < RG; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float fl = (float)clo[r][b], fh = (float)chi[r][b];
#pragma unroll
      for (int j = 0; j < NT8; ++j) {
        acc[r][j][0] = fmaf(fl, t[r][b][j][0], acc[r][j][0]);
        acc[r][j][1] = fmaf(fl, t[r][b][j][1], acc[r][j][1]);
        acc[r][j][2] = fmaf(fh, t[r][b][j][2], acc[r][j][2]);
        acc[r][j][3] = fmaf(fh, t[r][b][j][3], acc[r][j][3]);
      }
    }
}

template <int NT8, int CPC, int MODE>
__global__ void __launch_bounds__(DecCfg<NT8>::THREADS, 1)
    residual_dec_kernel(const DecParams p) {
  constexpr int NTOK = DecCfg<NT8>::NTOK;
  constexpr int PAR = DecCfg<NT8>::PAR;
  constexpr int CONSUMERS = DecCfg<NT8>::CONSUMERS;
  extern __shared__ __align__(128) unsigned char smem[];
  const int64_t D = p.D;
  const int nkb = (int)(D / 128);
  const int G = (int)(D >> p.g_shift);
  const int RR = p.r_c + p.r_r;
  const int SP = p.sp;
  const DecSmem m = dec_smem<NT8, MODE>(D, G, p.r_c, p.r_r, SP);
  const unsigned char* Hb = smem + m.h;
  const uint32_t corr_s = tc::smem_u32(smem + m.h + (size_t)NTOK * D * 2);
  unsigned char* pk = smem + m.pk;
  unsigned char* cds = smem + m.codes;
  int8_t* arc = reinterpret_cast<int8_t*>(smem + m.arow_c);
  int8_t* arw = reinterpret_cast<int8_t*>(smem + m.arow_w);
  float* ts = reinterpret_cast<float*>(smem + m.ts);  // ts[j * NTOK + n]
  unsigned char* ts16 = smem + m.ts16;
  const int tsb = (int)dec_ts16_stride(p.r_c + p.r_r);
  // rank terms on the tensor cores when both ranks are whole K=16 steps
  const bool rank_mma = (p.r_c % 16) == 0 && (p.r_r % 16) == 0;
  float2* red = reinterpret_cast<float2*>(smem + m.red);
  float4* xch = reinterpret_cast<float4*>(smem + m.xch);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + m.bars);
  uint64_t* h_full = bars;       // [1]
  uint64_t* c_full = bars + 1;   // [2]
  uint64_t* c_empty = bars + 3;  // [2]
  uint64_t* p_full = bars + 5;   // [SP]
  uint64_t* p_empty = p_full + SP;
  uint64_t* dead = p_empty + SP;  // test builds: a barrier nothing arrives on
  int* flag = reinterpret_cast<int*>(dead + 1);
  const int code_bytes = 128 * G;
  const size_t code_slot = dec_round16((size_t)code_bytes);
  const size_t arc_slot = dec_round16((size_t)128 * p.r_c);
  const size_t arw_slot = dec_round16((size_t)128 * p.r_r);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's units (tile, 128-column block), tile-major: [u0, u1)
  const int64_t U = p.n_vtiles * nkb, C = gridDim.x;
  const int64_t u0 = U * blockIdx.x / C, u1 = U * (blockIdx.x + 1) / C;

  if (threadIdx.x == 0) {
    tc::mbar_init(h_full, 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&c_full[s], 1);
      tc::mbar_init(&c_empty[s], CONSUMERS);
    }
    for (int s = 0; s < SP; ++s) {
      tc::mbar_init(&p_full[s], 1);
      tc::mbar_init(&p_empty[s], DecCfg<NT8>::WPP);  // the warps that take a stage
    }
    tc::mbar_init(dead, 1);
    tc::mbar_fence_init();
  }
  __syncthreads();

  if (warp == CONSUMERS) {
    // ---------------- producer (one thread) ----------------
    // A stage holds up to two consecutive blocks of one tile (contiguous in the device
    // layout, so one bulk copy).
    if (lane == 0) {
      bool ok = true;
      const uint64_t pol_first = tc::l2_policy_evict_first();  // the head streams once
      const uint32_t hbytes = (uint32_t)(NTOK * D * 2 + (int64_t)nkb * NTOK * 8 + NTOK * 4);
      // The H image comes from the prologue kernel, which may still be running (this
      // kernel is a programmatic dependent launch): the packed stream starts at once, and
      // the image is fetched after the prologue grid completes, before the first wait that
      // needs consumers to make progress.
      bool h_issued = false;
      auto issue_h = [&]() {
        if (h_issued) return;
        h_issued = true;
        grid_dependency_wait();
        tc::mbar_arrive_expect_tx(h_full, hbytes);
        tc::bulk_g2s(smem + m.h, p.Himg, hbytes, h_full);
      };
      int k = 0, np = 0, nc = 0, s = 0;
      for (int64_t u = u0; ok && u < u1; ++s) {
        const int64_t T = u / nkb;
        const int kb0 = (int)(u - T * nkb);
        const int kb1 = (int)((int64_t)nkb < kb0 + (u1 - u) ? (int64_t)nkb : kb0 + (u1 - u));
        const int cs = s & 1;
        if (s >= 2) issue_h();
        if (s >= 2 && !tc::mbar_wait(&c_empty[cs], ((s >> 1) - 1) & 1, p.err, p.wait_limit)) {
          ok = false;
          break;
        }
        tc::fence_proxy_async_smem();  // the slot was read with generic loads
        const int64_t row0 = T * 128;
        const int64_t rows = p.V - row0 < 128 ? p.V - row0 : 128;
        const bool acopy = dec_arow_copy(rows, p.r_c, p.r_r);
        const uint32_t abytes_c = acopy ? (uint32_t)(rows * p.r_c) : 0u;
        const uint32_t abytes_w = acopy ? (uint32_t)(rows * p.r_r) : 0u;
        tc::mbar_arrive_expect_tx(&c_full[cs], (uint32_t)code_bytes + abytes_c + abytes_w);
        tc::bulk_g2s(cds + cs * code_slot, p.code + row0 * G, (uint32_t)code_bytes, &c_full[cs]);
        if (abytes_c) tc::bulk_g2s(arc + cs * arc_slot, p.Ac + row0 * p.r_c, abytes_c, &c_full[cs]);
        if (abytes_w) tc::bulk_g2s(arw + cs * arw_slot, p.Aw + row0 * p.r_r, abytes_w, &c_full[cs]);
        ++nc;
        for (int kb = kb0; kb < kb1; kb += 2, ++k) {
          const int st = k % SP;
          const uint32_t bytes = (uint32_t)(kb + 1 < kb1 ? 2 * kDecPk : kDecPk);
          if (k >= SP) issue_h();
          if (k >= SP && !tc::mbar_wait(&p_empty[st], ((k / SP) - 1) & 1, p.err, p.wait_limit)) {
            ok = false;
            break;
          }
          tc::fence_proxy_async_smem();
          tc::mbar_arrive_expect_tx(&p_full[st], bytes);
          tc::bulk_g2s_hint(pk + (size_t)st * 2 * kDecPk, p.nib + ((T * nkb + kb) << 13), bytes,
                            &p_full[st], pol_first);
          ++np;
        }
        u += kb1 - kb0;
      }
      issue_h();
      tc::mbar_wait(h_full, 0, p.err, p.wait_limit);
      // Every copy this thread issued has landed before the CTA exits, whether or not the
      // consumers waited for it (after a timeout they stop waiting).  Each slot's last
      // issued phase is the one waited for here; in a normal run it has completed already.
      for (int q = np - SP < 0 ? 0 : np - SP; q < np; ++q)
        tc::mbar_wait(&p_full[q % SP], (q / SP) & 1, p.err, p.wait_limit);
      for (int q = nc - 2 < 0 ? 0 : nc - 2; q < nc; ++q)
        tc::mbar_wait(&c_full[q & 1], (q >> 1) & 1, p.err, p.wait_limit);
    }
    return;
  }

  // ---- consumers: warp w takes the stages k with k % PAR == w / WPP and owns the RG
  // 16-row groups RG (w % WPP) .. + RG - 1 of the tile ----
  constexpr int RG = DecCfg<NT8>::RG;
  constexpr int WPP = DecCfg<NT8>::WPP;
  const int gid = lane >> 2, tq = lane & 3;
  const int par = warp / WPP;
  const int wg = warp % WPP;
  const int ctid = threadIdx.x;  // 0 .. CONSUMERS * 32 - 1
  const int etid = wg * 32 + lane;  // the warps of parity 0 (which finish the tiles)
  grid_dependency_wait();  // t and the tile counters come from the prologue kernel
  bool ok = dec_wait(h_full, 0, p.err, true, p.wait_limit);
#ifdef ARCHEAD_TEST_HOOKS
  // failure-detection test: one warp waits on a barrier that never completes; its bounded
  // wait gives up, sets the device error word, and the warp skips its remaining waits
  if ((int)blockIdx.x == p.stall_cta && warp == 0) ok = dec_wait(dead, 0, p.err, ok, p.wait_limit);
#endif
  const float* tsc_s =
      reinterpret_cast<const float*>(smem + m.h + (size_t)NTOK * D * 2 + (size_t)nkb * NTOK * 8);
  for (int i = ctid; i < NTOK * RR; i += CONSUMERS * 32) {  // ts[j * NTOK + n]
    const int j = i / NTOK, n = i - j * NTOK;
    // t of the scaled token: t 2^-e_n (the token scales follow the image's corrections)
    const float tv = n < p.N ? __ldg(p.t + (int64_t)n * RR + j) / tsc_s[n] : 0.f;
    ts[i] = tv;
    // FP16 pieces: t1 + t2 carries 22 significant bits of t
    const __half t1 = __float2half_rn(tv);
    const __half t2 = __float2half_rn(tv - __half2float(t1));
    if (rank_mma && !(fabsf(tv) < 65504.f) && blockIdx.x == 0) atomicOr(p.err, kErrRangeH);
    *reinterpret_cast<__half*>(ts16 + n * tsb + j * 2) = t1;
    *reinterpret_cast<__half*>(ts16 + (NTOK + n) * tsb + j * 2) = t2;
  }
  asm volatile("bar.sync 10, %0;\n" ::"r"(CONSUMERS * 32) : "memory");

  const uint32_t pk_base = tc::smem_u32(pk);
  // ldmatrix row address of this lane for row group x: matrix lane / 8 = (chunk lane / 16,
  // row half (lane / 8) % 2), row lane % 8, plus 256 x; the second load takes chunks 2 and 3
  const uint32_t lm_off =
      (uint32_t)(((lane >> 4) * 128 + 16 * (RG * wg) + 8 * ((lane >> 3) & 1) + (lane & 7)) * 16);
  int r_lo[RG], r_hi[RG];
#pragma unroll
  for (int r = 0; r < RG; ++r) {
    r_lo[r] = 16 * (RG * wg + r) + gid;
    r_hi[r] = r_lo[r] + 8;
  }
  const float NEG_INF = __int_as_float(0xff800000);
  // B reads: byte offset of token 8j + gid's columns 32 tq + 8c of block kb in the
  // resident image is hrow[j] + 256 kb + hoff[c] (dec_h_offset unrolled)
  int hrow[NT8];
#pragma unroll
  for (int j = 0; j < NT8; ++j) hrow[j] = (8 * j + gid) * (int)D * 2 + 64 * tq;
  const int hx = (((tq >> 1) & 1) << 1) ^ (gid & 1);
  int hoff[4];
  uint32_t hoffu[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    hoff[c] = 16 * (c ^ hx);
    hoffu[c] = (uint32_t)hoff[c];
  }
  const uint32_t hs0 = tc::smem_u32(Hb) + (uint32_t)hrow[0];
  const uint32_t hj = (uint32_t)(8 * D * 2);
  const uint32_t cq0 = corr_s + (uint32_t)tq * 16;

  int k = 0, s = 0;
  bool nready = false;  // this warp's next stage, probed one stage ahead
  for (int64_t u = u0; u < u1; ++s) {
    const int64_t T = u / nkb;
    const int kb0 = (int)(u - T * nkb);
    const int kb1 = (int)((int64_t)nkb < kb0 + (u1 - u) ? (int64_t)nkb : kb0 + (u1 - u));
    const int cs = s & 1;
    const int64_t row0 = T * 128;
    ok = dec_wait(&c_full[cs], (s >> 1) & 1, p.err, ok, p.wait_limit);
    const unsigned char* crow_lo[RG];
    const unsigned char* crow_hi[RG];
#pragma unroll
    for (int r = 0; r < RG; ++r) {
      crow_lo[r] = cds + cs * code_slot + r_lo[r] * G;
      crow_hi[r] = cds + cs * code_slot + r_hi[r] * G;
    }

    float acc[RG][NT8][4];
#pragma unroll
    for (int r = 0; r < RG; ++r)
#pragma unroll
      for (int j = 0; j < NT8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[r][j][e] = 0.f;

    const int nst = (kb1 - kb0 + 1) >> 1;  // stages of this tile segment
    int i0 = (par - k % PAR + PAR) % PAR;  // this warp's first stage of them
    int st = (k + i0) % SP;
    uint32_t ph = (uint32_t)((k + i0) / SP) & 1u;
    k += nst;
    for (int i = i0; i < nst; i += PAR) {
      const int kb2 = kb0 + 2 * i;
      if (!nready) ok = ok && tc::mbar_wait(&p_full[st], ph, p.err, p.wait_limit);
      const int nb = kb2 + 1 < kb1 ? 2 : 1;
      uint32_t wlo[RG][2][4], whi[RG][2][4];  // [group][block][chunk]: word tq of rows r_lo, r_hi
      uint32_t clo[RG][2], chi[RG][2];
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        if (b < nb) {
          // group code of this thread's 32-column window (columns 32 tq .. 32 tq + 31)
          const int kb = kb2 + b;
          const int ci = CPC == 1 ? ((kb * 128) >> p.g_shift)
                                  : (CPC == 2 ? kb * 2 + (tq >> 1) : kb * 4 + tq);
#pragma unroll
          for (int r = 0; r < RG; ++r) {
            const uint32_t sa = pk_base + (uint32_t)(st * 2 + b) * kDecPk + lm_off + 256 * r;
            uint32_t q[4];
            ldmatrix_x4(sa, q);
            wlo[r][b][0] = q[0]; whi[r][b][0] = q[1]; wlo[r][b][1] = q[2]; whi[r][b][1] = q[3];
            ldmatrix_x4(sa + 2 * 128 * 16, q);
            wlo[r][b][2] = q[0]; whi[r][b][2] = q[1]; wlo[r][b][3] = q[2]; whi[r][b][3] = q[3];
            clo[r][b] = crow_lo[r][ci];
            chi[r][b] = crow_hi[r][ci];
          }
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_empty[st]);
      st += PAR;
      if (st >= SP) {
        st -= SP;
        ph ^= 1u;
      }
      nready = tc::mbar_test(&p_full[st], ph);
      if (CPC == 1) {
        const uint32_t hs = hs0 + (uint32_t)kb2 * 256u;
        const uint32_t cq = cq0 + (uint32_t)kb2 * (NTOK * 8);
        if (nb == 2)
          dec_blocks_q<NT8, 2, RG>(wlo, whi, clo, chi, hs, hj, hoffu, cq, acc);
        else
          dec_blocks_q<NT8, 1, RG>(wlo, whi, clo, chi, hs, hj, hoffu, cq, acc);
      } else {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          if (b >= nb) break;
          const int hb = (kb2 + b) * 256;
#pragma unroll
          for (int r = 0; r < RG; ++r) {
            const __half2 c2lo = __half2half2(__ushort2half_rn((unsigned short)clo[r][b]));
            const __half2 c2hi = __half2half2(__ushort2half_rn((unsigned short)chi[r][b]));
            const __half2 m24 = __float2half2_rn(-24.f);
            const __half2 n2lo = __hmul2(c2lo, m24), n2hi = __hmul2(c2hi, m24);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              __half2 pa[4], pb[4];
              dequant_word(wlo[r][b][c], c2lo, n2lo, pa);
              dequant_word(whi[r][b][c], c2hi, n2hi, pb);
              const uint32_t a0[4] = {h2_bits(pa[0]), h2_bits(pb[0]), h2_bits(pa[1]), h2_bits(pb[1])};
              const uint32_t a1[4] = {h2_bits(pa[2]), h2_bits(pb[2]), h2_bits(pa[3]), h2_bits(pb[3])};
#pragma unroll
              for (int j = 0; j < NT8; ++j) {
                const uint4 hv = *reinterpret_cast<const uint4*>(Hb + hrow[j] + hb + hoff[c]);
                mma_f16_16816(acc[r][j], a0, hv.x, hv.y);
                mma_f16_16816(acc[r][j], a1, hv.z, hv.w);
              }
            }
          }
        }
      }
    }

    // ---- warps of one row-group set: the warps of parity > 0 hand their sums to parity 0
    // (double-buffered by segment parity: parity 0 has read the buffers of segment s - 2
    // before it met the others at the barrier of segment s - 1) ----
    if (PAR > 1) {
      if (par) {
#pragma unroll
        for (int r = 0; r < RG; ++r) {
          float4* xs = xch + ((((size_t)(s & 1) * (PAR - 1) + par - 1) * 256) + (RG * wg + r) * 32 + lane) * NT8;
#pragma unroll
          for (int j = 0; j < NT8; ++j)
            xs[j] = make_float4(acc[r][j][0], acc[r][j][1], acc[r][j][2], acc[r][j][3]);
        }
      }
      asm volatile("bar.sync %0, %1;\n" ::"r"(2 + wg), "r"(32 * PAR) : "memory");
      if (par) {
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&c_empty[cs]);
        u += kb1 - kb0;
        continue;
      }
#pragma unroll
      for (int q2 = 1; q2 < PAR; ++q2)
#pragma unroll
        for (int r = 0; r < RG; ++r) {
          const float4* xs = xch + ((((size_t)(s & 1) * (PAR - 1) + q2 - 1) * 256) + (RG * wg + r) * 32 + lane) * NT8;
#pragma unroll
          for (int j = 0; j < NT8; ++j) {
            const float4 q = xs[j];
            acc[r][j][0] += q.x; acc[r][j][1] += q.y; acc[r][j][2] += q.z; acc[r][j][3] += q.w;
          }
        }
    }

    // ---- a tile split between CTAs: the last contributor to arrive finishes it ----
    bool finish = kb0 == 0 && kb1 == nkb;
    if (!finish) {
      const int slot = u == u0 ? 0 : 1;
#pragma unroll
      for (int r = 0; r < RG; ++r) {
        float4* dst = p.scratch + (((int64_t)blockIdx.x * 2 + slot) * 256 + (RG * wg + r) * 32 + lane) * NT8;
#pragma unroll
        for (int j = 0; j < NT8; ++j)
          dst[j] = make_float4(acc[r][j][0], acc[r][j][1], acc[r][j][2], acc[r][j][3]);
      }
      __threadfence();
      asm volatile("bar.sync 1, %0;\n" ::"r"(WPP * 32) : "memory");
      const int64_t cf = dec_cta_of(T * nkb, U, C), cl = dec_cta_of(T * nkb + nkb - 1, U, C);
      if (etid == 0) {
        const unsigned old = atomicAdd(p.counters + T, 1u);
        *flag = (int64_t)old + 1 == cl - cf + 1;
      }
      asm volatile("bar.sync 1, %0;\n" ::"r"(WPP * 32) : "memory");
      finish = *flag != 0;
      if (finish) {
        __threadfence();
#pragma unroll
        for (int r = 0; r < RG; ++r)
#pragma unroll
          for (int j = 0; j < NT8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[r][j][e] = 0.f;
        for (int64_t c = cf; c <= cl; ++c) {  // fixed order: the sum is deterministic
          const int64_t first_tile = (U * c / C) / nkb;
          const int sl = T == first_tile ? 0 : 1;
#pragma unroll
          for (int r = 0; r < RG; ++r) {
            const float4* src = p.scratch + ((c * 2 + sl) * 256 + (RG * wg + r) * 32 + lane) * NT8;
#pragma unroll
            for (int j = 0; j < NT8; ++j) {
              const float4 q = __ldcg(src + j);
              acc[r][j][0] += q.x; acc[r][j][1] += q.y; acc[r][j][2] += q.z; acc[r][j][3] += q.w;
            }
          }
        }
      }
    }

    if (finish) {
      // ---- epilogue: S_v acc + sAc Ac . t_c + sAw Aw . t_w, per row group ----
      const int64_t rows = p.V - row0 < 128 ? p.V - row0 : 128;
      const bool acopy = dec_arow_copy(rows, p.r_c, p.r_r);
#pragma unroll
      for (int r = 0; r < RG; ++r) {
        const int64_t v_lo = row0 + r_lo[r], v_hi = row0 + r_hi[r];
        const int64_t vc_lo = v_lo < p.V ? v_lo : p.V - 1, vc_hi = v_hi < p.V ? v_hi : p.V - 1;
        // row scales of the epilogue: the warps of parity 0 load them here while the others
        // already stream the next segment
        const float S_lo = bf16_bits_to_float(__ldg(p.sup + vc_lo));
        const float S_hi = bf16_bits_to_float(__ldg(p.sup + vc_hi));
        const float sac_lo = p.r_c ? __ldg(p.sAc + vc_lo) : 0.f, sac_hi = p.r_c ? __ldg(p.sAc + vc_hi) : 0.f;
        const float saw_lo = p.r_r ? __ldg(p.sAw + vc_lo) : 0.f, saw_hi = p.r_r ? __ldg(p.sAw + vc_hi) : 0.f;
        float y[NT8][4];
#pragma unroll
        for (int j = 0; j < NT8; ++j) {
          y[j][0] = S_lo * acc[r][j][0];
          y[j][1] = S_lo * acc[r][j][1];
          y[j][2] = S_hi * acc[r][j][2];
          y[j][3] = S_hi * acc[r][j][3];
        }
        if (rank_mma) {
          // [A_c | A_w] rows (INT8, exact in FP16) x FP16 hi / lo pieces of t, one FP32
          // accumulator per factor; thread q's K slots hold factor entries 16 s + 4 q + 0..3
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const int rank = part == 0 ? p.r_c : p.r_r;
            if (rank == 0) continue;
            const int8_t* abase = acopy ? (part == 0 ? arc + cs * arc_slot : arw + cs * arw_slot)
                                        : (part == 0 ? p.Ac : p.Aw);
            const int8_t* alo = abase + (acopy ? (int64_t)r_lo[r] : vc_lo) * rank;
            const int8_t* ahi = abase + (acopy ? (int64_t)r_hi[r] : vc_hi) * rank;
            const int off = part == 0 ? 0 : p.r_c;
            float L[NT8][4];
#pragma unroll
            for (int j = 0; j < NT8; ++j) L[j][0] = L[j][1] = L[j][2] = L[j][3] = 0.f;
            const __half2 k1152 = __float2half2_rn(1152.f);
            for (int st16 = 0; st16 < rank; st16 += 16) {
              const uint32_t wl = *reinterpret_cast<const uint32_t*>(alo + st16 + 4 * tq) ^ 0x80808080u;
              const uint32_t wh = *reinterpret_cast<const uint32_t*>(ahi + st16 + 4 * tq) ^ 0x80808080u;
              // bytes b + 128 under the FP16 pattern 0x6400 read 1024 + b + 128: minus 1152
              uint32_t q0 = __byte_perm(wl, 0x64646464u, 0x5140), q1 = __byte_perm(wl, 0x64646464u, 0x7352);
              uint32_t q2 = __byte_perm(wh, 0x64646464u, 0x5140), q3 = __byte_perm(wh, 0x64646464u, 0x7352);
              const uint32_t a[4] = {h2_bits(__hsub2(*reinterpret_cast<__half2*>(&q0), k1152)),
                                     h2_bits(__hsub2(*reinterpret_cast<__half2*>(&q2), k1152)),
                                     h2_bits(__hsub2(*reinterpret_cast<__half2*>(&q1), k1152)),
                                     h2_bits(__hsub2(*reinterpret_cast<__half2*>(&q3), k1152))};
#pragma unroll
              for (int pc = 0; pc < 2; ++pc)
#pragma unroll
                for (int j = 0; j < NT8; ++j) {
                  const uint2 bv = *reinterpret_cast<const uint2*>(
                      ts16 + (pc * NTOK + 8 * j + gid) * tsb + (off + st16 + 4 * tq) * 2);
                  mma_f16_16816(L[j], a, bv.x, bv.y);
                }
            }
            const float sl = part == 0 ? sac_lo : saw_lo, sh = part == 0 ? sac_hi : saw_hi;
#pragma unroll
            for (int j = 0; j < NT8; ++j) {
              y[j][0] = fmaf(sl, L[j][0], y[j][0]);
              y[j][1] = fmaf(sl, L[j][1], y[j][1]);
              y[j][2] = fmaf(sh, L[j][2], y[j][2]);
              y[j][3] = fmaf(sh, L[j][3], y[j][3]);
            }
          }
        } else {
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const int rank = part == 0 ? p.r_c : p.r_r;
            if (rank == 0) continue;
            const int8_t* abase = acopy ? (part == 0 ? arc + cs * arc_slot : arw + cs * arw_slot)
                                        : (part == 0 ? p.Ac : p.Aw);
            const int8_t* alo = abase + (acopy ? (int64_t)r_lo[r] : vc_lo) * rank;
            const int8_t* ahi = abase + (acopy ? (int64_t)r_hi[r] : vc_hi) * rank;
            const float* tcol = ts + (part == 0 ? 0 : p.r_c) * NTOK + 2 * tq;
            float llo[NT8][2], lhi[NT8][2];
#pragma unroll
            for (int j = 0; j < NT8; ++j) llo[j][0] = llo[j][1] = lhi[j][0] = lhi[j][1] = 0.f;
            auto step = [&](float al, float ah, int i) {
#pragma unroll
              for (int j = 0; j < NT8; ++j) {
                const float2 tv = *reinterpret_cast<const float2*>(tcol + i * NTOK + 8 * j);
                llo[j][0] = fmaf(al, tv.x, llo[j][0]);
                llo[j][1] = fmaf(al, tv.y, llo[j][1]);
                lhi[j][0] = fmaf(ah, tv.x, lhi[j][0]);
                lhi[j][1] = fmaf(ah, tv.y, lhi[j][1]);
              }
            };
            int i = 0;
            if ((rank & 3) == 0) {  // four INT8 entries per 32-bit load (rows 4-byte aligned)
              for (; i < rank; i += 4) {
                const uint32_t wl = *reinterpret_cast<const uint32_t*>(alo + i);
                const uint32_t wh = *reinterpret_cast<const uint32_t*>(ahi + i);
#pragma unroll
                for (int b = 0; b < 4; ++b)
                  step((float)(int8_t)(wl >> (8 * b)), (float)(int8_t)(wh >> (8 * b)), i + b);
              }
            }
            for (; i < rank; ++i) step((float)alo[i], (float)ahi[i], i);
            const float sl = part == 0 ? sac_lo : saw_lo, sh = part == 0 ? sac_hi : saw_hi;
#pragma unroll
            for (int j = 0; j < NT8; ++j) {
              y[j][0] = fmaf(sl, llo[j][0], y[j][0]);
              y[j][1] = fmaf(sl, llo[j][1], y[j][1]);
              y[j][2] = fmaf(sh, lhi[j][0], y[j][2]);
              y[j][3] = fmaf(sh, lhi[j][1], y[j][3]);
            }
          }
        }
        // the logits of the scaled tokens (8 j + 2 tq + e): times 2^e_n
#pragma unroll
        for (int j = 0; j < NT8; ++j) {
          const float2 tk = *reinterpret_cast<const float2*>(
              smem + m.h + (size_t)NTOK * D * 2 + (size_t)nkb * NTOK * 8 + (8 * j + 2 * tq) * 4);
          y[j][0] *= tk.x;
          y[j][1] *= tk.y;
          y[j][2] *= tk.x;
          y[j][3] *= tk.y;
        }
        if (MODE == 0) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int64_t v = h ? v_hi : v_lo;
            if (v >= p.V) continue;
#pragma unroll
            for (int j = 0; j < NT8; ++j)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int64_t tok = 8 * j + 2 * tq + e;
                if (tok < p.N) __stcs(p.Y + tok * p.V + v, y[j][2 * h + e]);
              }
          }
        } else {
          // ---- fused NLL: per token (max, sum exp) over the row group's rows, target logit ----
#pragma unroll
          for (int j = 0; j < NT8; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              float mx = NEG_INF;
              if (v_lo < p.V) mx = fmaxf(mx, y[j][e]);
              if (v_hi < p.V) mx = fmaxf(mx, y[j][2 + e]);
              float sm = 0.f;
              if (v_lo < p.V) sm += __expf(y[j][e] - mx);
              if (v_hi < p.V) sm += __expf(y[j][2 + e] - mx);
#pragma unroll
              for (int o = 4; o < 32; o <<= 1) {  // the 8 lanes sharing this token
                const float mo = __shfl_xor_sync(0xffffffffu, mx, o);
                const float so = __shfl_xor_sync(0xffffffffu, sm, o);
                const float mn = fmaxf(mx, mo);
                sm = (mx == NEG_INF ? 0.f : sm * __expf(mx - mn)) +
                     (mo == NEG_INF ? 0.f : so * __expf(mo - mn));
                mx = mn;
              }
              const int n = 8 * j + 2 * tq + e;
              if (gid == 0) red[(RG * wg + r) * NTOK + n] = make_float2(mx, sm);
              if (n < p.N) {
                const int64_t tgt = __ldg(p.targets + n);
                if (v_lo == tgt && v_lo < p.V) p.tlogit[n] = y[j][e];
                if (v_hi == tgt && v_hi < p.V) p.tlogit[n] = y[j][2 + e];
              }
            }
        }
      }
      if (MODE != 0) {
        // the tile's (max, sum exp) per token from its eight row groups
        asm volatile("bar.sync 1, %0;\n" ::"r"(WPP * 32) : "memory");
        for (int n = etid; n < NTOK; n += WPP * 32) {
          if (n >= p.N) continue;
          float mx = NEG_INF, sm = 0.f;
          for (int w = 0; w < kDecRows; ++w) {
            const float2 q = red[w * NTOK + n];
            const float mn = fmaxf(mx, q.x);
            sm = (mx == NEG_INF ? 0.f : sm * __expf(mx - mn)) +
                 (q.x == NEG_INF ? 0.f : q.y * __expf(q.x - mn));
            mx = mn;
          }
          p.part[(int64_t)n * p.n_vtiles + T] = make_float2(mx, sm);
        }
        asm volatile("bar.sync 1, %0;\n" ::"r"(WPP * 32) : "memory");
      }
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&c_empty[cs]);
    u += kb1 - kb0;
  }
}

template <int NT8, int CPC, int MODE>
cudaError_t launch_dec_cfg(const DecParams& p, int grid, cudaStream_t st) {
  const int G = (int)(p.D >> p.g_shift);
  const size_t smem = dec_smem<NT8, MODE>(p.D, G, p.r_c, p.r_r, p.sp).total;
  auto kern = residual_dec_kernel<NT8, CPC, MODE>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (p.sp % DecCfg<NT8>::PAR != 0) return cudaErrorInvalidValue;
  return launch_dependent(kern, grid, DecCfg<NT8>::THREADS, smem, st, p);
}

template <int NT8, int MODE>
cudaError_t launch_dec_nt(const DecParams& p, int g, int grid, cudaStream_t st) {
  if (g == 32) return launch_dec_cfg<NT8, 4, MODE>(p, grid, st);
  if (g == 64) return launch_dec_cfg<NT8, 2, MODE>(p, grid, st);
  return launch_dec_cfg<NT8, 1, MODE>(p, grid, st);
}

// The PAR warps of a row-group set take stages by the global stage index modulo PAR; with
// a ring of a multiple of PAR slots every use of a slot then goes to the same warps, which
// never wait on a slot's mbarrier more than one phase ahead (another count would let a
// fast warp skip a phase and alias the parity test).
template <int NT8, int MODE>
int fit_sp(const Shapes& s, size_t budget) {
  const int G = (int)(s.D / s.g);
  for (int sp = kDecMaxSP; sp >= 3; --sp)
    if (sp % DecCfg<NT8>::PAR == 0 &&
        dec_smem<NT8, MODE>(s.D, G, s.r_c, s.r_r, sp).total <= budget)
      return sp;
  return 0;
}

}  // namespace

#ifdef ARCHEAD_TEST_HOOKS
namespace {
long long g_hook_wait_limit = 1ll << 31;
int g_hook_stall_cta = -1;
}  // namespace
void set_dec_test_hooks(long long wait_limit, int stall_cta) {
  g_hook_wait_limit = wait_limit;
  g_hook_stall_cta = stall_cta;
}
#endif

DecPlan dec_plan(const Shapes& s, bool nll) {
  DecPlan pl = {0, 0, 0};
  if (s.N < 1 || s.N > 16) return pl;
  const size_t budget = 227 * 1024;  // one CTA per SM
  const int nt8 = s.N <= 8 ? 1 : 2;
  int sp;
  if (nt8 == 1) sp = nll ? fit_sp<1, 1>(s, budget) : fit_sp<1, 0>(s, budget);
  else sp = nll ? fit_sp<2, 1>(s, budget) : fit_sp<2, 0>(s, budget);
  if (!sp) return pl;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return pl;
  const int64_t units = (s.V + 127) / 128 * (s.D / 128);
  pl.nt8 = nt8;
  pl.sp = sp;
  pl.grid = (int)(units < sms ? units : sms);
  return pl;
}

size_t dec_image_bytes(const Shapes& s, const DecPlan& pl) {
  return (size_t)8 * pl.nt8 * s.D * 2 + (size_t)(s.D / 128) * 8 * pl.nt8 * 8 + (size_t)8 * pl.nt8 * 4;
}
size_t dec_partial_bytes(const DecPlan& pl) { return (size_t)pl.grid * 2 * 256 * pl.nt8 * 16; }

cudaError_t launch_dec_prologue(const uint16_t* H, const archead_head* head, const Shapes& s,
                                const DecPlan& pl, __half* img, float* t, unsigned* counters,
                                unsigned* err, cudaStream_t st, int* launches) {
  const int64_t ntok = 8 * pl.nt8;
  const int64_t n_counters = (s.V + 127) / 128;
  // one warp per (token, 128-column block), the counters on the same blocks; then one
  // block per factor index for t
  int64_t blocks = (ntok * (s.D / 128) * 32 + kDecPrologueThreads - 1) / kDecPrologueThreads;
  const int64_t cb = (n_counters + kDecPrologueThreads - 1) / kDecPrologueThreads;
  if (cb > blocks) blocks = cb;
  if (blocks > 148 * 8) blocks = 148 * 8;
  const int RR = s.r_c + s.r_r;
  dec_prologue_kernel<<<(unsigned)(blocks + RR), kDecPrologueThreads, 0, st>>>(
      H, img, s.N, (int)ntok, s.D, s.g >= 128 ? 1 : 0, counters, n_counters, (int)blocks,
      head->Bc, head->sBc, head->Bw, head->sBw, s.r_c, s.r_r, s.g, t, err);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_residual_dec(const __half* img, const float* t, const archead_head* head,
                                const Shapes& s, const DecPlan& pl, float* Y,
                                const int32_t* targets, float2* part, float* tlogit,
                                float4* scratch, unsigned* counters, unsigned* err,
                                cudaStream_t st, int* launches) {
  DecParams p;
  p.Himg = img;
  p.t = t;
  p.nib = head->r_nib;
  p.code = head->r_code;
  p.sup = head->r_super;
  p.Ac = head->Ac;
  p.sAc = head->sAc;
  p.Aw = head->Aw;
  p.sAw = head->sAw;
  p.Y = Y;
  p.targets = targets;
  p.part = part;
  p.tlogit = tlogit;
  p.scratch = scratch;
  p.counters = counters;
  p.N = s.N;
  p.V = s.V;
  p.D = s.D;
  p.r_c = s.r_c;
  p.r_r = s.r_r;
  int gs = 0;
  while ((1 << gs) < s.g) ++gs;
  p.g_shift = gs;
  p.sp = pl.sp;
  p.n_vtiles = (s.V + 127) / 128;
  p.err = err;
#ifdef ARCHEAD_TEST_HOOKS
  p.wait_limit = g_hook_wait_limit;
  p.stall_cta = g_hook_stall_cta;
#else
  p.wait_limit = 1ll << 31;
  p.stall_cta = -1;
#endif
  if (pl.nt8 < 1 || pl.nt8 > 2 || pl.sp < 3 || pl.sp > kDecMaxSP || pl.grid < 1)
    return cudaErrorInvalidValue;
  cudaError_t e;
  if (pl.nt8 == 1)
    e = Y ? launch_dec_nt<1, 0>(p, s.g, pl.grid, st) : launch_dec_nt<1, 1>(p, s.g, pl.grid, st);
  else
    e = Y ? launch_dec_nt<2, 0>(p, s.g, pl.grid, st) : launch_dec_nt<2, 1>(p, s.g, pl.grid, st);
  ++*launches;
  return e;
}

}  // namespace archead
