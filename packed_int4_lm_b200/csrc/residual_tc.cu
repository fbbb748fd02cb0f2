// Residual contraction on the 5th-generation tensor cores (tcgen05, TMEM accumulators).
//
//   Y[n, v] = S_v * sum_d h[n, d] q[v, d] c[v, d / g]  +  rank terms        (ARCHead Sec. 3)
//
// One CTA computes a 128-row vocabulary tile for a tile of NT tokens (NT = 16..128):
//  * warps 0-3 own one vocabulary row per thread (= one TMEM lane).  They stream the row's
//    packed nibbles (64 bytes per 128-column block, prefetched one block ahead),
//    dequantise them to exact FP16 q*c in registers and store them with tcgen05.st into a
//    two-stage A ring in tensor memory (a 128 x 128 FP16 block = 64 TMEM columns);
//  * warp 4, one thread: bulk-copies (TMA engine, no tensor map) the token tile's FP16 H
//    block -- pre-arranged by the prologue as the 8 x 16-byte core-matrix image the MMA
//    reads -- into a shared-memory ring;
//  * warp 5, one thread: issues tcgen05.mma kind::f16 with A from tensor memory and B from
//    shared memory, eight K=16 steps per block, into an M=128 x N=NT FP32 accumulator in
//    tensor memory, and commits each stage back to its producers;
//  * epilogue (warps 0-3): tcgen05.ld of the accumulator row, times S_v, plus the core and
//    correction rank terms from t staged in shared memory, stored coalesced into Y.
// Every mbarrier wait is bounded (about a second of SM cycles); a wait that gives up sets
// the device error word, the CTA drains what it issued and frees its tensor memory.
#include "tc_common.cuh"

namespace archead {
namespace {

constexpr int kTcThreads = 192;  // warps 0-3 dequant + epilogue, 4 H producer, 5 MMA issuer
constexpr int kASt = 2;          // A-ring stages in tensor memory (64 columns each)

struct TcParams {
  const __half* Hb;  // blocked FP16 H: [token tile][128-column block][NT x 128 image]
  const float* t;    // N x RR
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
  unsigned* err;
};

template <int NT>
struct TcCfg {
  static constexpr int SB = NT <= 64 ? 4 : 3;  // H ring stages
  static constexpr int HSTAGE = NT * 256;      // bytes of one 128-column H block
  static constexpr int TMEM_COLS = 256;        // NT accumulator columns + 2 x 64 A columns
  static_assert(NT + 64 * kASt <= TMEM_COLS, "tensor memory budget");
  static_assert(NT % 16 == 0 && NT >= 16 && NT <= 256, "M=128 MMA needs N in 16..256");
};

template <int NT>
size_t tc_smem_bytes(int RR) {
  using C = TcCfg<NT>;
  return (size_t)C::SB * C::HSTAGE + (size_t)RR * NT * 4 + 256;
}

// codes of the four 32-column windows of block kb (see residual_mma.cu: load_codes)
template <int CPC>
__device__ __forceinline__ void block_codes(const uint8_t* __restrict__ crow, int kb,
                                            int g_shift, uint32_t out[4]) {
  if (CPC == 1) {
    uint32_t c = __ldg(crow + ((kb * 128) >> g_shift));
    out[0] = out[1] = out[2] = out[3] = c;
  } else if (CPC == 2) {
    uint32_t c0 = __ldg(crow + kb * 2), c1 = __ldg(crow + kb * 2 + 1);
    out[0] = out[1] = c0;
    out[2] = out[3] = c1;
  } else {
#pragma unroll
    for (int w = 0; w < 4; ++w) out[w] = __ldg(crow + kb * 4 + w);
  }
}

template <int NT, int CPC>
__global__ void __launch_bounds__(kTcThreads, 1) residual_tc_kernel(const TcParams p) {
  using C = TcCfg<NT>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int RR = p.r_c + p.r_r;
  unsigned char* Hs = smem;
  float* ts = reinterpret_cast<float*>(smem + C::SB * C::HSTAGE);  // ts[j * NT + n]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SB * C::HSTAGE +
                                               (((size_t)RR * NT * 4 + 15) & ~(size_t)15));
  uint64_t* b_full = bars;
  uint64_t* b_empty = bars + C::SB;
  uint64_t* a_full = bars + 2 * C::SB;
  uint64_t* a_empty = a_full + kASt;
  uint64_t* acc_full = a_empty + kASt;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t D = p.D;
  const int nkb = (int)(D / 128);
  const int64_t row0 = (int64_t)blockIdx.y * 128;
  const int64_t tok0 = (int64_t)blockIdx.x * NT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SB; ++s) {
      tc::mbar_init(&b_full[s], 1);
      tc::mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < kASt; ++s) {
      tc::mbar_init(&a_full[s], 128);
      tc::mbar_init(&a_empty[s], 1);
    }
    tc::mbar_init(acc_full, 1);
    tc::mbar_fence_init();
  }
  if (warp == 5) tc::tmem_alloc(tmem_slot, C::TMEM_COLS);
  for (int i = threadIdx.x; i < NT * RR; i += kTcThreads) {
    const int j = i / NT, n = i - j * NT;
    const int64_t tok = tok0 + n;
    ts[i] = tok < p.N ? p.t[tok * RR + j] : 0.f;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  const uint32_t acol = tbase + NT;  // A ring: columns NT .. NT + 128 (lane field 0)

  if (warp == 4) {
    // ---------------- H producer ----------------
    if (lane == 0) {
      const unsigned char* src =
          reinterpret_cast<const unsigned char*>(p.Hb) + (int64_t)blockIdx.x * nkb * C::HSTAGE;
      int issued = 0;
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % C::SB;
        if (kb >= C::SB && !tc::mbar_wait(&b_empty[s], ((kb / C::SB) - 1) & 1, p.err)) {
          ok = false;
          break;
        }
        tc::mbar_arrive_expect_tx(&b_full[s], C::HSTAGE);
        tc::bulk_g2s(Hs + s * C::HSTAGE, src + (int64_t)kb * C::HSTAGE, C::HSTAGE, &b_full[s]);
        ++issued;
      }
      if (!ok) {  // drain copies that may still be in flight before the CTA exits
        for (int kb = issued - C::SB < 0 ? 0 : issued - C::SB; kb < issued; ++kb)
          tc::mbar_wait(&b_full[kb % C::SB], (kb / C::SB) & 1, p.err);
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_f16_m128(NT);
      for (int kb = 0; kb < nkb; ++kb) {
        const int sa = kb % kASt, sb = kb % C::SB;
        if (!tc::mbar_wait(&a_full[sa], (kb / kASt) & 1, p.err)) break;
        if (!tc::mbar_wait(&b_full[sb], (kb / C::SB) & 1, p.err)) break;
        tc::fence_after_sync();
        const uint32_t hb = tc::smem_u32(Hs + sb * C::HSTAGE);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint64_t bd = tc::smem_desc_kmajor(hb + 256 * j, 128, 2048);
          tc::mma_f16_ts(tbase, acol + 64 * sa + 8 * j, bd, idesc, (kb | j) != 0);
        }
        tc::mma_commit(&a_empty[sa]);
        tc::mma_commit(&b_empty[sb]);
      }
      tc::mma_commit(acc_full);
    }
  } else {
    // ---------------- dequant + epilogue: thread = vocabulary row = TMEM lane ----------------
    const int tid = threadIdx.x;  // 0..127
    const int64_t v = row0 + tid;
    const int64_t vc = v < p.V ? v : p.V - 1;  // tail rows load a valid row; results dropped
    const uint8_t* nrow = p.nib + vc * (D / 2);
    const uint8_t* crow = p.code + vc * (D >> p.g_shift);
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    bool ok = true;

    uint4 cur[4], nxt[4];
    uint32_t cc[4], cn[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) cur[i] = ldg_stream(nrow + 16 * i);
    block_codes<CPC>(crow, 0, p.g_shift, cc);

    for (int kb = 0; kb < nkb; ++kb) {
      const int sa = kb % kASt;
      if (kb + 1 < nkb) {
#pragma unroll
        for (int i = 0; i < 4; ++i) nxt[i] = ldg_stream(nrow + (int64_t)(kb + 1) * 64 + 16 * i);
        block_codes<CPC>(crow, kb + 1, p.g_shift, cn);
      }
      // 16 words: slot 4t + w holds block columns 32w + 8t + {0..7}; its pair i is
      // A columns (32w + 8t + 2i, +1) = TMEM column 16w + 4t + i of this stage
      uint32_t a[64];
      const uint32_t wds[16] = {cur[0].x, cur[0].y, cur[0].z, cur[0].w, cur[1].x, cur[1].y,
                                cur[1].z, cur[1].w, cur[2].x, cur[2].y, cur[2].z, cur[2].w,
                                cur[3].x, cur[3].y, cur[3].z, cur[3].w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const __half2 c2 = __half2half2(__ushort2half_rn((unsigned short)cc[w]));
        const __half2 nc24 = __hmul2(c2, __float2half2_rn(-24.f));
#pragma unroll
        for (int t4 = 0; t4 < 4; ++t4) {
          __half2 pr[4];
          dequant_word(wds[4 * t4 + w], c2, nc24, pr);
#pragma unroll
          for (int i = 0; i < 4; ++i) a[16 * w + 4 * t4 + i] = h2_bits(pr[i]);
        }
      }
      if (kb >= kASt) {
        // warp-uniform outcome: the tcgen05 stores below are whole-warp instructions
        if (!__all_sync(0xffffffffu, tc::mbar_wait(&a_empty[sa], ((kb / kASt) - 1) & 1, p.err))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
      }
      const uint32_t ta = acol + 64 * sa + lane_off;
      tc::tmem_st16(ta, a);
      tc::tmem_st16(ta + 16, a + 16);
      tc::tmem_st16(ta + 32, a + 32);
      tc::tmem_st16(ta + 48, a + 48);
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&a_full[sa]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        cur[i] = nxt[i];
        cc[i] = cn[i];
      }
    }

    if (ok && __all_sync(0xffffffffu, tc::mbar_wait(acc_full, 0, p.err))) {
      tc::fence_after_sync();
      const float S = bf16_bits_to_float(__ldg(p.sup + vc));
      const float sac = p.r_c ? __ldg(p.sAc + vc) : 0.f;
      const float saw = p.r_r ? __ldg(p.sAw + vc) : 0.f;
      const int8_t* arow_c = p.Ac + vc * p.r_c;
      const int8_t* arow_w = p.Aw + vc * p.r_r;
#pragma unroll 1
      for (int c = 0; c < NT / 16; ++c) {
        float y[16];
        tc::tmem_ld16(tbase + lane_off + 16 * c, y);
#pragma unroll
        for (int k = 0; k < 16; ++k) y[k] *= S;
#pragma unroll 1
        for (int part = 0; part < 2; ++part) {
          const int rank = part == 0 ? p.r_c : p.r_r;
          if (rank == 0) continue;
          const int8_t* arow = part == 0 ? arow_c : arow_w;
          const float* tcol = ts + (part == 0 ? 0 : p.r_c) * NT + 16 * c;
          float lr[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) lr[k] = 0.f;
          for (int j = 0; j < rank; ++j) {
            const float aj = (float)__ldg(arow + j);
            const float4* tp = reinterpret_cast<const float4*>(tcol + j * NT);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 tv = tp[q];
              lr[4 * q + 0] = fmaf(aj, tv.x, lr[4 * q + 0]);
              lr[4 * q + 1] = fmaf(aj, tv.y, lr[4 * q + 1]);
              lr[4 * q + 2] = fmaf(aj, tv.z, lr[4 * q + 2]);
              lr[4 * q + 3] = fmaf(aj, tv.w, lr[4 * q + 3]);
            }
          }
          const float sc = part == 0 ? sac : saw;
#pragma unroll
          for (int k = 0; k < 16; ++k) y[k] = fmaf(sc, lr[k], y[k]);
        }
        if (v < p.V) {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int64_t tok = tok0 + 16 * c + k;
            if (tok < p.N) p.Y[tok * p.V + v] = y[k];
          }
        }
      }
    }
  }

  if (warp == 5 && lane == 0) tc::mbar_wait(acc_full, 0, p.err);  // all MMAs retired
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// FP16 copy of H in the blocked image the MMA's B operand reads: for token tile tt of NT
// rows and 128-column block kb, a contiguous NT x 128 block whose 16-byte piece (token n,
// columns 8c..8c+7) sits at ((n / 8) * 16 + c) * 128 + (n % 8) * 16 bytes.  Rows >= N are
// zero.  Non-finite or out-of-range FP16 values set kErrRangeH.
__global__ void __launch_bounds__(256) convert_h_blocked_kernel(const uint16_t* __restrict__ H,
                                                                __half* __restrict__ Hb,
                                                                int64_t N, int64_t Npad,
                                                                int64_t D, int nt,
                                                                unsigned* err) {
  const int64_t chunks_per_row = D / 8;
  const int64_t total = Npad * chunks_per_row;
  const int64_t nkb = D / 128;
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = i / chunks_per_row;
    const int64_t kc = i - n * chunks_per_row;
    uint4 out = make_uint4(0, 0, 0, 0);
    if (n < N) {
      const uint4 in = *reinterpret_cast<const uint4*>(H + n * D + kc * 8);
      const uint32_t w[4] = {in.x, in.y, in.z, in.w};
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __half2 h = __floats2half2_rn(__uint_as_float(w[k] << 16),
                                            __uint_as_float(w[k] & 0xFFFF0000u));
        o[k] = h2_bits(h);
        bad |= ((o[k] & 0x7C00u) == 0x7C00u) | ((o[k] & 0x7C000000u) == 0x7C000000u);
      }
      out = make_uint4(o[0], o[1], o[2], o[3]);
    }
    const int64_t tt = n / nt, nn = n - tt * nt;
    const int64_t kb = kc >> 4, c = kc & 15;
    const int64_t off = (tt * nkb + kb) * (int64_t)nt * 128 + ((nn >> 3) * 16 + c) * 64 + (nn & 7) * 8;
    *reinterpret_cast<uint4*>(Hb + off) = out;
  }
  if (bad) atomicOr(err, kErrRangeH);
}

template <int NT, int CPC>
cudaError_t launch_tc_cfg(const TcParams& p, cudaStream_t st) {
  const int RR = p.r_c + p.r_r;
  const size_t smem = tc_smem_bytes<NT>(RR);
  auto kern = residual_tc_kernel<NT, CPC>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.N + NT - 1) / NT), (unsigned)((p.V + 127) / 128));
  kern<<<grid, kTcThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <int NT>
cudaError_t launch_tc_nt(const TcParams& p, int g, cudaStream_t st) {
  if (g == 32) return launch_tc_cfg<NT, 4>(p, st);
  if (g == 64) return launch_tc_cfg<NT, 2>(p, st);
  return launch_tc_cfg<NT, 1>(p, st);
}

}  // namespace

int tc_token_tile(int64_t N, int RR) {
  if (N <= 16) return 16;
  if (N <= 32) return 32;
  if (N <= 64 || RR > 128) return 64;
  return 128;
}

cudaError_t launch_prologue_blocked(const uint16_t* H, const archead_head* head,
                                    const Shapes& s, int nt, __half* Hb, float* t,
                                    unsigned* err, cudaStream_t st, int* launches) {
  const int64_t Npad = (s.N + nt - 1) / nt * nt;
  int64_t blocks = (Npad * s.D / 8 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  convert_h_blocked_kernel<<<(unsigned)(blocks < 1 ? 1 : blocks), 256, 0, st>>>(
      H, Hb, s.N, Npad, s.D, nt, err);
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_lowrank_t(H, head, s, t, st, launches);
}

cudaError_t launch_residual_tc(const __half* Hb, const float* t, const archead_head* head,
                               const Shapes& s, float* Y, unsigned* err, cudaStream_t st,
                               int* launches) {
  TcParams p;
  p.Hb = Hb;
  p.t = t;
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
  p.err = err;
  const int nt = tc_token_tile(s.N, s.r_c + s.r_r);
  cudaError_t e;
  switch (nt) {
    case 16: e = launch_tc_nt<16>(p, s.g, st); break;
    case 32: e = launch_tc_nt<32>(p, s.g, st); break;
    case 64: e = launch_tc_nt<64>(p, s.g, st); break;
    default: e = launch_tc_nt<128>(p, s.g, st); break;
  }
  ++*launches;
  return e;
}

}  // namespace archead
