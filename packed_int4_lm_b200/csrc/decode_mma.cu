// Small-batch decode (N <= 16) of the ARCHead logit path on warp-level tensor cores:
//
//   Y[n, v] = S_v * sum_d h[n, d] q[v, d] c[v, d / g]  +  rank terms        (ARCHead Sec. 3)
//
// Memory-bound: every packed byte is read from HBM once per call, and the work per byte is
// a handful of integer/FP16 instructions (dequantisation) plus a few MMAs, so the kernel
// is built for bytes in flight and independent warps:
//  * every warp owns a contiguous run of R-tile row groups (16 rows per tile) -- the same
//    number of tiles for every warp -- and never synchronises with other warps;
//  * each thread streams its rows' packed 16-byte pieces with cp.async into a private
//    DEP-deep slot ring in shared memory (the warp's 16 rows x 64 bytes per 128-column
//    block are one contiguous kilobyte, so copies and reads are conflict free); the pipeline
//    loop is unrolled by DEP so that no register holding an in-flight load is ever copied;
//  * the A fragments are the raw offset-binary nibbles under the FP16 exponent of 1024, i.e.
//    1032 + q, made with three shifts and four LOP3 per eight weights and no FP16 work.
//    Each scale group accumulates into a temporary, and at the group's end
//        acc += c * (tmp - 1032 * sum_{d in group} h[n, d])
//    with the per-token group sums of H precomputed (exact FP16 products, FP32 sums);
//  * the FP16 hidden states (N x D, L1-resident) are read as B fragments from global memory;
//  * after a tile's last block: S_v, the core and correction rank terms from t in shared
//    memory, and the Y stores, while the next tile's blocks are already in flight.
#include "archead_internal.cuh"

namespace archead {
namespace {

struct DecParams {
  const __half* Hh;    // Npad x D, row-major FP16 (zero rows beyond N)
  const float* t;      // N x RR
  const float* hsum;   // N x G: 1032 * sum of H over each group
  const uint8_t* nib;
  const uint8_t* code;
  const uint16_t* sup;
  const int8_t* Ac;
  const float* sAc;
  const int8_t* Aw;
  const float* sAw;
  float* Y;
  int64_t N, V, D;
  int r_c, r_r, g_shift;
  int tiles_per_warp;  // R-tile groups per warp
};

// hsum[n, k] = 1032 * sum_{d in group k} h[n, d]: one warp per (token, group).
__global__ void __launch_bounds__(256) hsum_kernel(const uint16_t* __restrict__ H,
                                                   float* __restrict__ hsum, int64_t N,
                                                   int64_t D, int g) {
  const int64_t G = D / g;
  const int lane = threadIdx.x & 31;
  for (int64_t wi = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; wi < N * G;
       wi += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int64_t n = wi / G, k = wi - n * G;
    const uint16_t* row = H + n * D + k * g;
    float acc = 0.f;
    for (int i = lane; i < g; i += 32) acc += bf16_bits_to_float(row[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) hsum[wi] = 1032.f * acc;
  }
}

constexpr int kDecWarps = 4;

template <int R, int DEP>
struct DecCfg {
  static constexpr int SLOT = R * 2 * 32 * 16;  // bytes per warp per ring slot
  static constexpr int WARP_RING = DEP * SLOT;
};

template <int CPC>
__device__ __forceinline__ void load_codes_raw(const uint8_t* __restrict__ crow, int kb,
                                               int g_shift, uint32_t out[4]) {
  if (CPC == 1) {
    out[0] = __ldg(crow + ((kb * 128) >> g_shift));
  } else if (CPC == 2) {
    out[0] = __ldg(crow + kb * 2);
    out[1] = __ldg(crow + kb * 2 + 1);
  } else {
#pragma unroll
    for (int w = 0; w < 4; ++w) out[w] = __ldg(crow + kb * 4 + w);
  }
}

template <int CPC>
__device__ __forceinline__ uint32_t code_of_window(const uint32_t c[4], int w) {
  return CPC == 1 ? c[0] : (CPC == 2 ? c[w >> 1] : c[w]);
}

template <int NT, int R, int GW, int DEP>
__global__ void __launch_bounds__(kDecWarps * 32, 4) decode_mma_kernel(const DecParams p) {
  constexpr int CPC = GW >= 4 ? 1 : 4 / GW;  // code bytes per 128-column block
  using C = DecCfg<R, DEP>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tq = lane & 3;
  const int RR = p.r_c + p.r_r;
  const int TS = RR + 1;  // padded: the four token columns of a warp hit four banks
  constexpr int NTOK = NT * 8;
  unsigned char* ring = smem + warp * C::WARP_RING;
  float* ts = reinterpret_cast<float*>(smem + kDecWarps * C::WARP_RING);
  float* hs = ts + NTOK * TS;  // hs[k * NTOK + n]
  const int64_t D = p.D;
  const int G = (int)(D >> p.g_shift);

  for (int i = threadIdx.x; i < NTOK * RR; i += kDecWarps * 32) {
    const int n = i / RR, j = i - n * RR;
    ts[n * TS + j] = n < p.N ? p.t[n * RR + j] : 0.f;
  }
  for (int i = threadIdx.x; i < NTOK * G; i += kDecWarps * 32) {
    const int k = i / NTOK, n = i - k * NTOK;
    hs[i] = n < p.N ? p.hsum[(int64_t)n * G + k] : 0.f;
  }
  __syncthreads();

  const int nkb = (int)(D / 128);
  const int64_t gw = (int64_t)blockIdx.x * kDecWarps + warp;
  const int64_t grp0 = gw * p.tiles_per_warp;  // first R-tile group of this warp
  const int total = p.tiles_per_warp * nkb;    // blocks this warp streams

  // ---- issue side: (group, block) of the next block to copy ----
  int iss_g = 0, iss_kb = 0;
  uint32_t cq[DEP][R][2][4];
  auto issue = [&](int slot, uint32_t (&codes)[R][2][4]) {
    unsigned char* dst = ring + slot * C::SLOT + lane * 16;
    if (iss_g < p.tiles_per_warp) {
      const int64_t vbase = (grp0 + iss_g) * (16 * R);
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t v = vbase + 16 * r + gid + 8 * h;
          const bool live = v < p.V;
          const int64_t vc = live ? v : 0;
          cp_async16_zfill(dst + (r * 2 + h) * 512,
                           p.nib + nib_chunk_offset(vc, iss_kb, nkb, tq),
                           live ? 16u : 0u);
          load_codes_raw<CPC>(p.code + vc * (D >> p.g_shift), iss_kb, p.g_shift, codes[r][h]);
        }
      if (++iss_kb == nkb) {
        iss_kb = 0;
        ++iss_g;
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int q = 0; q < DEP - 1; ++q) issue(q, cq[q]);

  float acc[R][NT][4], tmp[R][NT][4];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[r][j][e] = tmp[r][j][e] = 0.f;

  // B fragments (four 32-column windows x NT token tiles) of block kb, read through L1 one
  // block ahead of their use (ping-pong by the parity of the unrolled step)
  static_assert(DEP % 2 == 0, "B-fragment ping-pong needs an even ring depth");
  uint4 bfq[2][4][NT];
  auto load_b = [&](int kbl, uint4 (&dst)[4][NT]) {
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
      for (int j = 0; j < NT; ++j)
        dst[w][j] = __ldg(reinterpret_cast<const uint4*>(
            p.Hh + (int64_t)(8 * j + gid) * D + (int64_t)kbl * 128 + 32 * w + 8 * tq));
  };
  load_b(0, bfq[0]);

  int kb = 0, grp = 0;
  for (int k0 = 0; k0 < total; k0 += DEP) {
#pragma unroll
    for (int u = 0; u < DEP; ++u) {
      // a predicate, not a break: the loop must unroll fully so ring indices stay static
      issue((u + DEP - 1) % DEP, cq[(u + DEP - 1) % DEP]);
      if (k0 + u < total) {
      load_b(kb + 1 == nkb ? 0 : kb + 1, bfq[(u + 1) & 1]);
      const uint4 (&bf)[4][NT] = bfq[u & 1];
      cp_async_wait<DEP - 1>();
      const unsigned char* src = ring + u * C::SLOT + lane * 16;
      uint4 pk[R][2];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          pk[r][h] = *reinterpret_cast<const uint4*>(src + (r * 2 + h) * 512);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          uint32_t x[2][4];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t word = w == 0 ? pk[r][h].x : w == 1 ? pk[r][h].y
                                                      : w == 2 ? pk[r][h].z : pk[r][h].w;
            magic_word(word, x[h]);
          }
          const uint32_t a0[4] = {x[0][0], x[1][0], x[0][1], x[1][1]};
          const uint32_t a1[4] = {x[0][2], x[1][2], x[0][3], x[1][3]};
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            mma_f16_16816(tmp[r][j], a0, bf[w][j].x, bf[w][j].y);
            mma_f16_16816(tmp[r][j], a1, bf[w][j].z, bf[w][j].w);
          }
        }
        // end of a scale group: acc += c * (tmp - 1032 * group sum of H)
        if (GW > 4 ? (w == 3 && (kb & 1)) : ((w + 1) % GW == 0)) {
          const int grp_k = (kb * 4 + w) / GW;
          float hsv[NT][2];
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            const float2 v2 = *reinterpret_cast<const float2*>(hs + grp_k * NTOK + 8 * j + 2 * tq);
            hsv[j][0] = v2.x;
            hsv[j][1] = v2.y;
          }
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float c = (float)code_of_window<CPC>(cq[u][r][h], w);
#pragma unroll
              for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  acc[r][j][2 * h + e] = fmaf(c, tmp[r][j][2 * h + e] - hsv[j][e],
                                              acc[r][j][2 * h + e]);
                  tmp[r][j][2 * h + e] = 0.f;
                }
            }
        }
      }
      if (++kb == nkb) {
        // ---- epilogue of row group grp: S_v * acc + rank terms, store ----
        const int64_t vbase = (grp0 + grp) * (16 * R);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int64_t v = vbase + 16 * r + gid + 8 * h;
            if (v >= p.V) continue;
            const float S = bf16_bits_to_float(__ldg(p.sup + v));
            float y[NT][2];
#pragma unroll
            for (int j = 0; j < NT; ++j) {
              y[j][0] = S * acc[r][j][2 * h];
              y[j][1] = S * acc[r][j][2 * h + 1];
            }
#pragma unroll 1
            for (int part = 0; part < 2; ++part) {
              const int rank = part == 0 ? p.r_c : p.r_r;
              if (rank == 0) continue;
              const int8_t* arow = (part == 0 ? p.Ac : p.Aw) + v * rank;
              const float sa = __ldg((part == 0 ? p.sAc : p.sAw) + v);
              const int off = part == 0 ? 0 : p.r_c;
              float lr[NT][2];
#pragma unroll
              for (int j = 0; j < NT; ++j) lr[j][0] = lr[j][1] = 0.f;
              auto acc_i = [&](float a, int i) {
#pragma unroll
                for (int j = 0; j < NT; ++j)
#pragma unroll
                  for (int e = 0; e < 2; ++e)
                    lr[j][e] = fmaf(a, ts[(8 * j + 2 * tq + e) * TS + off + i], lr[j][e]);
              };
              int i = 0;
              if ((rank & 3) == 0 && (reinterpret_cast<uintptr_t>(arow) & 3) == 0) {
                const uint32_t* a4 = reinterpret_cast<const uint32_t*>(arow);
#pragma unroll 2
                for (; i < rank; i += 4) {
                  const uint32_t wv = __ldg(a4 + (i >> 2));
                  acc_i((float)(int8_t)(wv & 0xFF), i);
                  acc_i((float)(int8_t)((wv >> 8) & 0xFF), i + 1);
                  acc_i((float)(int8_t)((wv >> 16) & 0xFF), i + 2);
                  acc_i((float)(int8_t)(wv >> 24), i + 3);
                }
              }
              for (; i < rank; ++i) acc_i((float)__ldg(arow + i), i);
#pragma unroll
              for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) y[j][e] = fmaf(sa, lr[j][e], y[j][e]);
            }
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int64_t tok = 8 * j + 2 * tq + e;
                if (tok < p.N) p.Y[tok * p.V + v] = y[j][e];
              }
          }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[r][j][e] = 0.f;
        kb = 0;
        ++grp;
      }
      }
    }
  }
  cp_async_wait<0>();
}

template <int NT, int R, int GW, int DEP>
cudaError_t launch_dec_cfg(const DecParams& p0, cudaStream_t st) {
  using C = DecCfg<R, DEP>;
  DecParams p = p0;
  const int RR = p.r_c + p.r_r;
  const int G = (int)(p.D >> p.g_shift);
  const size_t smem = (size_t)kDecWarps * C::WARP_RING + (size_t)NT * 8 * (RR + 1) * 4 +
                      (size_t)NT * 8 * G * 4;
  auto kern = decode_mma_kernel<NT, R, GW, DEP>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, occ = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kDecWarps * 32, smem)) !=
      cudaSuccess)
    return e;
  if (occ < 1) occ = 1;
  // every warp gets the same number of R-tile groups, and all warps are resident at once
  const int64_t groups = (p.V + 16 * R - 1) / (16 * R);
  const int64_t slots = (int64_t)sms * occ * kDecWarps;
  p.tiles_per_warp = (int)((groups + slots - 1) / slots);
  const int64_t warps = (groups + p.tiles_per_warp - 1) / p.tiles_per_warp;
  const int64_t blocks = (warps + kDecWarps - 1) / kDecWarps;
  kern<<<(unsigned)blocks, kDecWarps * 32, smem, st>>>(p);
  return cudaGetLastError();
}

template <int NT, int R, int DEP>
cudaError_t launch_dec_g(const DecParams& p, int g, cudaStream_t st) {
  if (g == 32) return launch_dec_cfg<NT, R, 1, DEP>(p, st);
  if (g == 64) return launch_dec_cfg<NT, R, 2, DEP>(p, st);
  if (g == 128) return launch_dec_cfg<NT, R, 4, DEP>(p, st);
  return launch_dec_cfg<NT, R, 8, DEP>(p, st);
}

}  // namespace

cudaError_t launch_decode_mma(const uint16_t* H, const __half* Hh, const float* t,
                              float* hsum, const archead_head* head, const Shapes& s,
                              float* Y, cudaStream_t st, int* launches) {
  {
    const int64_t warps = s.N * (s.D / s.g);
    int64_t blocks = (warps * 32 + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    hsum_kernel<<<(unsigned)(blocks < 1 ? 1 : blocks), 256, 0, st>>>(H, hsum, s.N, s.D, s.g);
    ++*launches;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  DecParams p;
  p.Hh = Hh;
  p.t = t;
  p.hsum = hsum;
  p.nib = head->r_nib;
  p.code = head->r_code;
  p.sup = head->r_super;
  p.Ac = head->Ac;
  p.sAc = head->sAc;
  p.Aw = head->Aw;
  p.sAw = head->sAw;
  p.Y = Y;
  p.N = s.N;
  p.V = s.V;
  p.D = s.D;
  p.r_c = s.r_c;
  p.r_r = s.r_r;
  int gs = 0;
  while ((1 << gs) < s.g) ++gs;
  p.g_shift = gs;
  p.tiles_per_warp = 1;
  cudaError_t e = s.N <= 8 ? launch_dec_g<1, 2, 4>(p, s.g, st)
                           : launch_dec_g<2, 1, 4>(p, s.g, st);
  ++*launches;
  return e;
}

}  // namespace archead
