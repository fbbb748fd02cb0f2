// Residual contraction of the ARCHead logit path with its low-rank epilogue:
//
//   Y[n, v] = S_v * sum_d h[n, d] q[v, d] c[v, d / g]                 (SC4 residual, Sec. 3)
//           + sAc[v] * sum_j Ac[v, j] t[n, j]                         (quantized core)
//           + sAw[v] * sum_j Aw[v, j] t[n, r_c + j]                   (correction, Sec. 3)
//
// (ARCHead Sec. 3: Y = H W_d^T + (H B_w^T) A_w^T with W_d = Q8(A_c) Q8(B_c) + SC4(R).)
//
// Warp-level tensor-core path (mma.sync m16n8k16, FP16 operands, FP32 accumulators):
//  * each warp owns R tiles of 16 vocabulary rows and streams their packed nibbles with
//    128-bit non-allocating loads (one 16-byte chunk per thread and row from the tiled
//    device layout), prefetched one 128-column chunk ahead in registers;
//    every packed byte is read from HBM once per token block;
//  * nibbles are dequantised in registers to q * c (exact in FP16) straight into the A
//    fragment; the device nibble layout makes one 32-bit word feed two k16 steps;
//  * the token block's FP16 hidden states (the B operand) are staged in shared memory by
//    cp.async in a 3-stage ring, XOR-swizzled so the 128-bit fragment reads are
//    conflict-free;
//  * the epilogue applies S_v and adds the rank terms from t staged in shared memory.
// MODE 0 writes Y.  MODE 1 (fused NLL) writes, per token and vocabulary block, the
// (max, sum of exp(y - max)) pair and the target's logit, and never writes Y.  MODE 2
// (agreement with a dense reference head, Sec. 5 Table 8) writes, per token and vocabulary
// block, the packed (max, sum exp), the dense (max, sum exp, argmax), the KL accumulator
// sum exp(y_d - max_d) (y_d - y_p) and the block's k largest packed logits with their ids;
// agreement_merge_kernel combines the blocks.
#include "archead_internal.cuh"

namespace archead {
namespace {

constexpr int kKC = 128;     // columns per pipeline chunk (one 64-byte block of a row)
constexpr int kStages = 3;   // cp.async ring depth for the hidden-state chunks

struct GemmParams {
  const __half* Hh;  // Npad x D (token n scaled by 2^-e_n)
  const float* t;    // N x RR (scaled the same way)
  const float* tsc;  // N token scales 2^e_n
  const uint8_t* nib;        // SC4: tiled nibbles; Row INT8 (CPC = 0): V x D int8 row-major
  const float* row_scale;    // Row INT8: W[v, d] = q8[v, d] * row_scale[v]
  const uint8_t* code;
  const uint16_t* sup;
  const int8_t* Ac;
  const float* sAc;
  const int8_t* Aw;
  const float* sAw;
  float* Y;
  const int32_t* targets;
  float2* part;
  float* tlogit;
  int64_t N, V, D;
  int r_c, r_r, g_shift;
  int nvblk;
  int red_off;  // byte offset of the MODE 1 reduction buffer in dynamic shared memory
  // MODE 2
  const float* Yd;  // N x V dense reference logits
  int topk;         // 1..kAgreeMaxK
  float* astat;     // [N][nvblk][6]: m_p, s_p, m_d, s_d, kl accumulator, dense argmax (bits)
  float* akval;     // [N][nvblk][topk] largest packed logits of the block, decreasing
  int* akid;        // [N][nvblk][topk] their vocabulary ids (-1 past the last row)
};

constexpr int kAgreeMaxK = 16;

// Order of the agreement top-k: larger value first, equal values by smaller id.
__device__ __forceinline__ bool agree_better(float a, int ia, float b, int ib) {
  return a > b || (a == b && (unsigned)ia < (unsigned)ib);
}

constexpr int kRows = 128;  // vocabulary rows per block in every configuration

template <int NT, int R, int WARPS>
struct Cfg {
  static constexpr int NTOK = NT * 8;
  static constexpr int ROWS = 16 * R * WARPS;
  static constexpr int THREADS = WARPS * 32;
  static constexpr int HS_BYTES = kStages * NTOK * kKC * 2;
};

// Codes for the 4 windows of chunk kc of one row (CPC codes per chunk, g = 128 / CPC for
// CPC > 1, g >= 128 otherwise; CPC = 0 is the Row INT8 format, which has none).
template <int CPC>
__device__ __forceinline__ void load_codes(const uint8_t* __restrict__ crow, int kc,
                                           int g_shift, uint32_t out[4]) {
  if (CPC == 0) {
    out[0] = out[1] = out[2] = out[3] = 0u;
  } else if (CPC == 1) {
    uint32_t c = __ldg(crow + ((kc * kKC) >> g_shift));
    out[0] = out[1] = out[2] = out[3] = c;
  } else if (CPC == 2) {
    uint32_t c0 = __ldg(crow + kc * 2), c1 = __ldg(crow + kc * 2 + 1);
    out[0] = out[1] = c0;
    out[2] = out[3] = c1;
  } else {
#pragma unroll
    for (int w = 0; w < 4; ++w) out[w] = __ldg(crow + kc * 4 + w);
  }
}

template <int NT, int R, int WARPS, int CPC, int MODE>
__global__ void __launch_bounds__(WARPS * 32)
    residual_mma_kernel(const GemmParams p) {
  using C = Cfg<NT, R, WARPS>;
  static_assert(C::ROWS == kRows, "block row count");
  extern __shared__ __align__(128) unsigned char smem[];
  __half* Hs = reinterpret_cast<__half*>(smem);

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int gid = lane >> 2;  // row within the 8-row half tile / token within n8 tile
  const int tq = lane & 3;    // thread within quad
  const int64_t D = p.D;
  const int nchunks = (int)(D / kKC);
  // grid.x walks token blocks so that blocks sharing vocabulary rows run back to back
  // and re-read the packed rows from L2 rather than HBM when there are several
  const int64_t row_block = (int64_t)blockIdx.y * C::ROWS;
  const int64_t tok0 = (int64_t)blockIdx.x * C::NTOK;

  // rows owned by this thread: tile r -> rows base + gid and base + gid + 8
  int64_t vrow[R][2];
  const uint8_t* nib_row[R][2];
  const uint8_t* code_row[R][2];
#pragma unroll
  for (int r = 0; r < R; ++r) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      int64_t v = row_block + (int64_t)(warp * R + r) * 16 + gid + 8 * h;
      vrow[r][h] = v;
      int64_t vc = v < p.V ? v : p.V - 1;  // clamp loads of tail rows; results discarded
      // SC4: chunk tq of the row's block 0 in the tiled layout; Row INT8: the 8 bytes of
      // columns 8 tq .. 8 tq + 7 of the row (window w adds 32 w, chunk kc adds 128 kc)
      nib_row[r][h] = CPC == 0 ? p.nib + vc * D + 8 * tq
                               : p.nib + nib_chunk_offset(vc, 0, D / 128, tq);
      code_row[r][h] = CPC == 0 ? p.nib : p.code + vc * (D >> p.g_shift);
    }
  }

  // hidden-state chunk loader: NTOK rows x 128 columns -> 16-byte pieces, swizzled
  auto load_h = [&](int kc, int stage) {
    __half* dst = Hs + (size_t)stage * C::NTOK * kKC;
    constexpr int PIECES = C::NTOK * (kKC / 8);
    for (int i = threadIdx.x; i < PIECES; i += C::THREADS) {
      int n = i >> 4, c = i & 15;
      int cs = c ^ ((n & 1) << 2);
      cp_async16(dst + n * kKC + cs * 8, p.Hh + (tok0 + n) * D + (int64_t)kc * kKC + c * 8);
    }
  };

  float acc[R][NT][4];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[r][j][e] = 0.f;

  // pipeline prologue
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < nchunks) load_h(s, s);
    cp_async_commit();
  }
  // words of the current chunk: SC4 one 16-byte chunk (word w = window w), Row INT8 four
  // 8-byte pieces (words 2w, 2w + 1 = window w)
  constexpr int NW = CPC == 0 ? 8 : 4;
  auto load_chunk = [&](const uint8_t* row, int kc, uint32_t out[NW]) {
    if (CPC == 0) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint2 x = ldg_stream8(row + (int64_t)kc * kKC + 32 * w);
        out[(2 * w) % NW] = x.x;
        out[(2 * w + 1) % NW] = x.y;
      }
    } else {
      const uint4 x = ldg_stream(row + ((int64_t)kc << 13));
      out[0] = x.x;
      out[1 % NW] = x.y;
      out[2 % NW] = x.z;
      out[3 % NW] = x.w;
    }
  };
  uint32_t cur[R][2][NW];
  uint32_t ccur[R][2][4];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      load_chunk(nib_row[r][h], 0, cur[r][h]);
      load_codes<CPC>(code_row[r][h], 0, p.g_shift, ccur[r][h]);
    }

  for (int kc = 0; kc < nchunks; ++kc) {
    __syncthreads();  // all warps are done with the stage that is refilled below
    {
      int nk = kc + kStages - 1;
      if (nk < nchunks) load_h(nk, nk % kStages);
      cp_async_commit();
    }
    uint32_t nxt[R][2][NW];
    uint32_t cnxt[R][2][4];
    const bool more = kc + 1 < nchunks;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (more) {
          load_chunk(nib_row[r][h], kc + 1, nxt[r][h]);
          load_codes<CPC>(code_row[r][h], kc + 1, p.g_shift, cnxt[r][h]);
        } else {
#pragma unroll
          for (int w = 0; w < NW; ++w) nxt[r][h][w] = 0;
#pragma unroll
          for (int w = 0; w < 4; ++w) cnxt[r][h][w] = 0;
        }
      }
    cp_async_wait<kStages - 1>();
    __syncthreads();

    const __half* hs = Hs + (size_t)(kc % kStages) * C::NTOK * kKC;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint4 bf[NT];
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        int n = 8 * j + gid;
        int cs = (4 * w + tq) ^ ((gid & 1) << 2);
        bf[j] = *reinterpret_cast<const uint4*>(hs + n * kKC + cs * 8);
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        __half2 pr[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (CPC == 0) {
            // INT8 bytes (columns 0..7 of the window) as exact FP16 pairs: b + 128 under
            // the pattern 0x6400 reads 1024 + b + 128, minus 1152
            const __half2 k1152 = __float2half2_rn(1152.f);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const uint32_t x = cur[r][h][(2 * w + q) % NW] ^ 0x80808080u;
              uint32_t q0 = __byte_perm(x, 0x64646464u, 0x5140);
              uint32_t q1 = __byte_perm(x, 0x64646464u, 0x7352);
              pr[h][2 * q] = __hsub2(*reinterpret_cast<__half2*>(&q0), k1152);
              pr[h][2 * q + 1] = __hsub2(*reinterpret_cast<__half2*>(&q1), k1152);
            }
          } else {
            const uint32_t word = cur[r][h][w % NW];
            __half2 c2 = __half2half2(__ushort2half_rn((unsigned short)ccur[r][h][w]));
            __half2 nc24 = __hmul2(c2, __float2half2_rn(-24.f));
            dequant_word(word, c2, nc24, pr[h]);
          }
        }
        uint32_t a0[4] = {h2_bits(pr[0][0]), h2_bits(pr[1][0]), h2_bits(pr[0][1]),
                          h2_bits(pr[1][1])};
        uint32_t a1[4] = {h2_bits(pr[0][2]), h2_bits(pr[1][2]), h2_bits(pr[0][3]),
                          h2_bits(pr[1][3])};
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          mma_f16_16816(acc[r][j], a0, bf[j].x, bf[j].y);
          mma_f16_16816(acc[r][j], a1, bf[j].z, bf[j].w);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int w = 0; w < NW; ++w) cur[r][h][w] = nxt[r][h][w];
#pragma unroll
        for (int w = 0; w < 4; ++w) ccur[r][h][w] = cnxt[r][h][w];
      }
  }
  cp_async_wait<0>();
  __syncthreads();  // the hidden-state ring is reused for t below

  // ---- epilogue: S_v * acc + rank terms ----
  const int RR = p.r_c + p.r_r;
  float* ts = reinterpret_cast<float*>(smem);
  const int TS = RR + 1;  // padded stride: the 4 token columns of a warp hit 4 banks
  for (int i = threadIdx.x; i < C::NTOK * RR; i += C::THREADS) {
    int n = i / RR, j = i - n * RR;
    int64_t tok = tok0 + n;
    ts[n * TS + j] = tok < p.N ? p.t[tok * RR + j] : 0.f;
  }
  for (int n = threadIdx.x; n < C::NTOK; n += C::THREADS)  // column RR: the token scale
    ts[n * TS + RR] = tok0 + n < p.N ? p.tsc[tok0 + n] : 1.f;
  __syncthreads();

  float y[R][NT][4];
#pragma unroll
  for (int r = 0; r < R; ++r) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t v = vrow[r][h];
      const int64_t vc = v < p.V ? v : p.V - 1;
      const float S = CPC == 0 ? __ldg(p.row_scale + vc) : bf16_bits_to_float(__ldg(p.sup + vc));
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) y[r][j][2 * h + e] = S * acc[r][j][2 * h + e];
      // core and correction rank terms, each with its own row scale
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const int rank = part == 0 ? p.r_c : p.r_r;
        if (rank == 0) continue;
        const int8_t* arow = (part == 0 ? p.Ac : p.Aw) + vc * rank;
        const float sa = __ldg((part == 0 ? p.sAc : p.sAw) + vc);
        const int off = part == 0 ? 0 : p.r_c;
        float lr[NT][2];
#pragma unroll
        for (int j = 0; j < NT; ++j) lr[j][0] = lr[j][1] = 0.f;
        for (int i = 0; i < rank; ++i) {
          const float a = (float)__ldg(arow + i);
#pragma unroll
          for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e)
              lr[j][e] = fmaf(a, ts[(8 * j + 2 * tq + e) * TS + off + i], lr[j][e]);
        }
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) y[r][j][2 * h + e] = fmaf(sa, lr[j][e], y[r][j][2 * h + e]);
      }
      // the logits of the scaled tokens: times 2^e_n
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) y[r][j][2 * h + e] *= ts[(8 * j + 2 * tq + e) * TS + RR];
    }
  }

  if (MODE == 2) {
    // ---- agreement: the block's packed and dense tiles in shared memory, then one warp
    // per token reduces its 128 rows ----
    constexpr int LD = kRows + 1;
    __syncthreads();  // t is no longer read: the buffer becomes the two tiles
    float* yp = reinterpret_cast<float*>(smem);  // [NTOK][LD] packed logits
    float* yd = yp + C::NTOK * LD;              // [NTOK][LD] dense logits
    const float NEG_INF = __int_as_float(0xff800000);
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int lr = (warp * R + r) * 16 + gid + 8 * h;
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            yp[(8 * j + 2 * tq + e) * LD + lr] = vrow[r][h] < p.V ? y[r][j][2 * h + e] : NEG_INF;
      }
    for (int i = threadIdx.x; i < C::NTOK * kRows; i += C::THREADS) {
      const int n = i / kRows, lr = i - n * kRows;
      const int64_t v = row_block + lr, tok = tok0 + n;
      yd[n * LD + lr] = v < p.V && tok < p.N ? __ldg(p.Yd + tok * p.V + v) : NEG_INF;
    }
    __syncthreads();
    for (int n = warp; n < C::NTOK; n += WARPS) {
      const int64_t tok = tok0 + n;
      if (tok >= p.N) break;  // uniform over the warp; later tokens are past N too
      float a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = yp[n * LD + lane + 32 * q];
        b[q] = yd[n * LD + lane + 32 * q];
      }
      // packed and dense maxima (dense argmax: the smallest row among equal maxima)
      float mp = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
      float md = NEG_INF;
      int ad = 0x7fffffff;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (agree_better(b[q], lane + 32 * q, md, ad)) {
          md = b[q];
          ad = lane + 32 * q;
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mp = fmaxf(mp, __shfl_xor_sync(0xffffffffu, mp, o));
        const float mo = __shfl_xor_sync(0xffffffffu, md, o);
        const int ao = __shfl_xor_sync(0xffffffffu, ad, o);
        if (agree_better(mo, ao, md, ad)) {
          md = mo;
          ad = ao;
        }
      }
      float sp = 0.f, sd = 0.f, kl = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (a[q] != NEG_INF) sp += __expf(a[q] - mp);
        if (b[q] != NEG_INF) {
          const float w = __expf(b[q] - md);
          sd += w;
          kl = fmaf(w, b[q] - a[q], kl);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sp += __shfl_xor_sync(0xffffffffu, sp, o);
        sd += __shfl_xor_sync(0xffffffffu, sd, o);
        kl += __shfl_xor_sync(0xffffffffu, kl, o);
      }
      const int64_t rec = tok * p.nvblk + blockIdx.y;
      if (lane == 0) {
        float* st = p.astat + rec * 6;
        st[0] = mp;
        st[1] = sp;
        st[2] = md;
        st[3] = sd;
        st[4] = kl;
        st[5] = __int_as_float(md == NEG_INF ? -1 : (int)(row_block + ad));
      }
      // the block's topk largest packed logits: topk rounds of a warp argmax; the winner's
      // lane retires that entry
      for (int i = 0; i < p.topk; ++i) {
        float bv = NEG_INF;
        int bi = 0x7fffffff;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (agree_better(a[q], lane + 32 * q, bv, bi)) {
            bv = a[q];
            bi = lane + 32 * q;
          }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float vo = __shfl_xor_sync(0xffffffffu, bv, o);
          const int io = __shfl_xor_sync(0xffffffffu, bi, o);
          if (agree_better(vo, io, bv, bi)) {
            bv = vo;
            bi = io;
          }
        }
        if (bv != NEG_INF && (bi & 31) == lane) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (lane + 32 * q == bi) a[q] = NEG_INF;
        }
        if (lane == 0) {
          p.akval[rec * p.topk + i] = bv;
          p.akid[rec * p.topk + i] = bv == NEG_INF ? -1 : (int)(row_block + bi);
        }
      }
    }
    return;
  }

  if (MODE == 0) {
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t v = vrow[r][h];
        if (v >= p.V) continue;
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int64_t tok = tok0 + 8 * j + 2 * tq + e;
            if (tok < p.N) p.Y[tok * p.V + v] = y[r][j][2 * h + e];
          }
      }
    return;
  }

  // ---- MODE 1: per-token (max, sum exp) over this block's rows, and the target logit ----
  float2* red = reinterpret_cast<float2*>(smem + p.red_off);  // [WARPS][NTOK]
  const float NEG_INF = __int_as_float(0xff800000);
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float m = NEG_INF;
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (vrow[r][h] < p.V) m = fmaxf(m, y[r][j][2 * h + e]);
      float sum = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (vrow[r][h] < p.V) sum += __expf(y[r][j][2 * h + e] - m);
      // combine the 8 lanes that share this token (same tq, different gid)
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o);
        const float so = __shfl_xor_sync(0xffffffffu, sum, o);
        const float mn = fmaxf(m, mo);
        const float a = (m == NEG_INF) ? 0.f : sum * __expf(m - mn);
        const float b = (mo == NEG_INF) ? 0.f : so * __expf(mo - mn);
        sum = a + b;
        m = mn;
      }
      const int n = 8 * j + 2 * tq + e;
      if (gid == 0) red[warp * C::NTOK + n] = make_float2(m, sum);
      const int64_t tok = tok0 + n;
      if (tok < p.N) {
        const int64_t tgt = __ldg(p.targets + tok);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (vrow[r][h] == tgt && vrow[r][h] < p.V) p.tlogit[tok] = y[r][j][2 * h + e];
      }
    }
  __syncthreads();
  for (int n = threadIdx.x; n < C::NTOK; n += C::THREADS) {
    const int64_t tok = tok0 + n;
    if (tok >= p.N) continue;
    float m = NEG_INF, sum = 0.f;
    for (int w = 0; w < WARPS; ++w) {
      const float2 q = red[w * C::NTOK + n];
      const float mn = fmaxf(m, q.x);
      const float a = (m == NEG_INF) ? 0.f : sum * __expf(m - mn);
      const float b = (q.x == NEG_INF) ? 0.f : q.y * __expf(q.x - mn);
      sum = a + b;
      m = mn;
    }
    p.part[tok * p.nvblk + blockIdx.y] = make_float2(m, sum);
  }
}

// nll[n] = M + log(sum_b s_b exp(m_b - M)) - y_target, one warp per token, fixed order.
__global__ void __launch_bounds__(256) nll_combine_kernel(const float2* __restrict__ part,
                                                          const float* __restrict__ tlogit,
                                                          const int32_t* __restrict__ targets,
                                                          int64_t N, int64_t V, int nvblk,
                                                          float* __restrict__ nll,
                                                          unsigned* err) {
  const int lane = threadIdx.x & 31;
  const int64_t n = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (n >= N) return;
  const float NEG_INF = __int_as_float(0xff800000);
  const float2* pr = part + n * nvblk;
  float m = NEG_INF;
  for (int b = lane; b < nvblk; b += 32) m = fmaxf(m, pr[b].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float s = 0.f;
  for (int b = lane; b < nvblk; b += 32) {
    const float2 q = pr[b];
    if (q.x != NEG_INF) s += q.y * expf(q.x - m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    const int32_t tg = targets[n];
    if (tg < 0 || (int64_t)tg >= V) {
      nll[n] = __int_as_float(0x7fc00000);
      atomicOr(err, kErrTarget);
    } else {
      nll[n] = m + logf(s) - tlogit[n];
    }
  }
}

template <int NT, int R, int WARPS, int CPC, int MODE>
cudaError_t launch_cfg(const GemmParams& p0, cudaStream_t st) {
  using C = Cfg<NT, R, WARPS>;
  GemmParams p = p0;
  const int RR = p.r_c + p.r_r;
  size_t ts = (size_t)C::NTOK * (RR + 1) * 4;
  if (MODE == 2) {  // the packed and dense tiles of the agreement epilogue
    const size_t tiles = (size_t)2 * C::NTOK * (kRows + 1) * 4;
    ts = ts > tiles ? ts : tiles;
  }
  size_t base = (size_t)C::HS_BYTES > ts ? (size_t)C::HS_BYTES : ts;
  base = (base + 15) & ~(size_t)15;
  p.red_off = (int)base;
  const size_t smem = base + (size_t)WARPS * C::NTOK * sizeof(float2);
  auto kern = residual_mma_kernel<NT, R, WARPS, CPC, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.N + C::NTOK - 1) / C::NTOK), (unsigned)p.nvblk);
  kern<<<grid, C::THREADS, smem, st>>>(p);
  return cudaGetLastError();
}

template <int NT, int R, int WARPS, int MODE>
cudaError_t launch_cpc(const GemmParams& p, int g, cudaStream_t st) {
  if (p.row_scale) return launch_cfg<NT, R, WARPS, 0, MODE>(p, st);  // Row INT8
  if (g == 32) return launch_cfg<NT, R, WARPS, 4, MODE>(p, st);
  if (g == 64) return launch_cfg<NT, R, WARPS, 2, MODE>(p, st);
  return launch_cfg<NT, R, WARPS, 1, MODE>(p, st);
}

template <int MODE>
cudaError_t launch_mode(const GemmParams& p, int g, cudaStream_t st) {
  if (p.N <= 8) return launch_cpc<1, 2, 4, MODE>(p, g, st);
  if (p.N <= 16) return launch_cpc<2, 2, 4, MODE>(p, g, st);
  if (p.N <= 32) return launch_cpc<4, 1, 8, MODE>(p, g, st);
  return launch_cpc<8, 1, 8, MODE>(p, g, st);
}

}  // namespace

int64_t residual_token_block(int64_t N) {
  if (N <= 8) return 8;
  if (N <= 16) return 16;
  if (N <= 32) return 32;
  return 64;
}

int residual_gemm_vblocks(const Shapes& s) { return (int)((s.V + kRows - 1) / kRows); }

cudaError_t launch_residual_gemm(const __half* Hh, const float* t, const float* tsc,
                                 const archead_head* head,
                                 const Shapes& s, float* Y, const int32_t* targets,
                                 float2* part, float* tlogit, cudaStream_t st, int* launches,
                                 int mode) {
  GemmParams p;
  p.Hh = Hh;
  p.t = t;
  p.tsc = tsc;
  p.nib = head->r_nib;
  p.row_scale = head->format == ARCHEAD_FMT_ROW8 ? head->row_scale : nullptr;
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
  p.N = s.N;
  p.V = s.V;
  p.D = s.D;
  p.r_c = s.r_c;
  p.r_r = s.r_r;
  int gs = 0;
  while ((1 << gs) < s.g) ++gs;
  p.g_shift = gs;
  p.nvblk = residual_gemm_vblocks(s);
  p.red_off = 0;
  p.Yd = nullptr;
  p.topk = 0;
  p.astat = p.akval = nullptr;
  p.akid = nullptr;
  cudaError_t e = mode == 0 ? launch_mode<0>(p, s.g, st) : launch_mode<1>(p, s.g, st);
  ++*launches;
  return e;
}

// Per token, one warp: the blocks' records are taken lane by lane in block order and
// combined with a fixed shuffle tree (deterministic).  Each lane keeps a sorted list of the
// best kAgreeMaxK candidates of its blocks; the warp then draws the topk best by repeated
// warp argmax.
__global__ void __launch_bounds__(256) agreement_merge_kernel(
    const float* __restrict__ astat, const float* __restrict__ akval,
    const int* __restrict__ akid, int64_t N, int nvblk, int topk, int32_t* __restrict__ topk_out,
    int32_t* __restrict__ top1_dense, float* __restrict__ kl_out, float* __restrict__ lse_out) {
  const int lane = threadIdx.x & 31;
  const int64_t n = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (n >= N) return;
  const float NEG_INF = __int_as_float(0xff800000);
  float mp = NEG_INF, sp = 0.f, md = NEG_INF, sd = 0.f, kl = 0.f;
  int ad = 0x7fffffff;
  float kv[kAgreeMaxK];
  int ki[kAgreeMaxK];
#pragma unroll
  for (int i = 0; i < kAgreeMaxK; ++i) {
    kv[i] = NEG_INF;
    ki[i] = 0x7fffffff;
  }
  auto merge_p = [&](float m2, float s2) {
    const float mn = fmaxf(mp, m2);
    sp = (mp == NEG_INF ? 0.f : sp * expf(mp - mn)) + (m2 == NEG_INF ? 0.f : s2 * expf(m2 - mn));
    mp = mn;
  };
  auto merge_d = [&](float m2, float s2, float k2, int a2) {
    const float mn = fmaxf(md, m2);
    const float f1 = md == NEG_INF ? 0.f : expf(md - mn), f2 = m2 == NEG_INF ? 0.f : expf(m2 - mn);
    sd = sd * f1 + s2 * f2;
    kl = kl * f1 + k2 * f2;
    if (agree_better(m2, a2, md, ad)) ad = a2;
    md = mn;
  };
  for (int b = lane; b < nvblk; b += 32) {
    const int64_t rec = n * nvblk + b;
    const float* st = astat + rec * 6;
    merge_p(st[0], st[1]);
    merge_d(st[2], st[3], st[4], __float_as_int(st[5]));
    for (int i = 0; i < topk; ++i) {
      float cv = akval[rec * topk + i];
      int ci = akid[rec * topk + i];
      if (cv == NEG_INF || !agree_better(cv, ci, kv[kAgreeMaxK - 1], ki[kAgreeMaxK - 1])) break;
#pragma unroll
      for (int j = 0; j < kAgreeMaxK; ++j)  // insertion: the carried entry swaps down
        if (agree_better(cv, ci, kv[j], ki[j])) {
          const float tv = kv[j];
          const int ti = ki[j];
          kv[j] = cv;
          ki[j] = ci;
          cv = tv;
          ci = ti;
        }
    }
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    merge_p(__shfl_xor_sync(0xffffffffu, mp, o), __shfl_xor_sync(0xffffffffu, sp, o));
    const float m2 = __shfl_xor_sync(0xffffffffu, md, o), s2 = __shfl_xor_sync(0xffffffffu, sd, o);
    const float k2 = __shfl_xor_sync(0xffffffffu, kl, o);
    const int a2 = __shfl_xor_sync(0xffffffffu, ad, o);
    merge_d(m2, s2, k2, a2);
  }
  // topk rounds: every lane offers the head of its list, the best one is drawn
  int head = 0;
  for (int i = 0; i < topk; ++i) {
    float bv = NEG_INF;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < kAgreeMaxK; ++j)
      if (j == head) {
        bv = kv[j];
        bi = ki[j];
      }
    float wv = bv;
    int wi = bi;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float vo = __shfl_xor_sync(0xffffffffu, wv, o);
      const int io = __shfl_xor_sync(0xffffffffu, wi, o);
      if (agree_better(vo, io, wv, wi)) {
        wv = vo;
        wi = io;
      }
    }
    if (wv != NEG_INF && wi == bi && wv == bv) ++head;  // this lane's head was drawn
    if (lane == 0) topk_out[n * topk + i] = wv == NEG_INF ? -1 : wi;
  }
  if (lane == 0) {
    const float lp = mp + logf(sp), ld = md + logf(sd);
    top1_dense[n] = ad == 0x7fffffff ? -1 : ad;
    kl_out[n] = kl / sd - ld + lp;
    if (lse_out) lse_out[n] = lp;
  }
}

cudaError_t launch_agreement(const __half* Hh, const float* t, const float* tsc,
                             const archead_head* head,
                             const Shapes& s, const float* Yd, int topk, float* astat,
                             float* akval, int* akid, int32_t* topk_out, int32_t* top1_dense,
                             float* kl_out, float* lse_out, cudaStream_t st, int* launches) {
  GemmParams p;
  p.Hh = Hh;
  p.t = t;
  p.tsc = tsc;
  p.nib = head->r_nib;
  p.row_scale = head->format == ARCHEAD_FMT_ROW8 ? head->row_scale : nullptr;
  p.code = head->r_code;
  p.sup = head->r_super;
  p.Ac = head->Ac;
  p.sAc = head->sAc;
  p.Aw = head->Aw;
  p.sAw = head->sAw;
  p.Y = nullptr;
  p.targets = nullptr;
  p.part = nullptr;
  p.tlogit = nullptr;
  p.N = s.N;
  p.V = s.V;
  p.D = s.D;
  p.r_c = s.r_c;
  p.r_r = s.r_r;
  int gs = 0;
  while ((1 << gs) < s.g) ++gs;
  p.g_shift = gs;
  p.nvblk = residual_gemm_vblocks(s);
  p.red_off = 0;
  p.Yd = Yd;
  p.topk = topk;
  p.astat = astat;
  p.akval = akval;
  p.akid = akid;
  if (topk < 1 || topk > kAgreeMaxK) return cudaErrorInvalidValue;
  cudaError_t e = launch_mode<2>(p, s.g, st);
  ++*launches;
  if (e != cudaSuccess) return e;
  agreement_merge_kernel<<<(unsigned)((s.N + 7) / 8), 256, 0, st>>>(
      astat, akval, akid, s.N, p.nvblk, topk, topk_out, top1_dense, kl_out, lse_out);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_nll_combine(const float2* part, const float* tlogit,
                               const int32_t* targets, const Shapes& s, float* nll,
                               unsigned* err, cudaStream_t st, int* launches) {
  const int nvblk = residual_gemm_vblocks(s);
  nll_combine_kernel<<<(unsigned)((s.N + 7) / 8), 256, 0, st>>>(part, tlogit, targets, s.N,
                                                                 s.V, nvblk, nll, err);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace archead
