// Residual contraction on the 5th-generation tensor cores (tcgen05, TMEM accumulators).
//
//   Y[n, v] = S_v * sum_d h[n, d] q[v, d] c[v, d / g]  +  rank terms        (ARCHead Sec. 3)
//
// Persistent, warp-specialised kernel.  A work item is one 128-row vocabulary tile for one
// tile of NT tokens (NT = 16..128):
//  * warp 8 (two threads, independent streams) feeds three shared-memory rings with bulk
//    copies (TMA engine, no tensor map, no multicast): the tile's 8 KB packed-nibble block
//    per 128 columns (the
//    tiled device layout makes it one contiguous region), the tile's group-scale codes once
//    per item, and the token tile's FP16 H block (pre-arranged by the prologue as the
//    128-byte-swizzled K-major image the MMA reads);
//  * warps 0-3 (dequant): one vocabulary row per thread (= one TMEM lane).  A thread reads
//    its row's four 16-byte chunks of the block (conflict free: chunk i of row s sits at
//    (i * 128 + s) * 16), dequantises them to exact FP16 q*c and stores them with
//    tcgen05.st into an A ring of 2-4 stages in tensor memory (128 x 128 FP16 = 64
//    columns per stage); the dequant warps issue no global loads;
//  * warp 9 (one thread): issues tcgen05.mma kind::f16, A from tensor memory, B from
//    shared memory, eight K=16 steps per block, into one of two M=128 x N=NT FP32
//    accumulators, so the next item's MMAs overlap the previous item's epilogue;
//  * warps 4-7 (epilogue): tcgen05.ld of an accumulator row, times S_v, plus the core and
//    correction rank terms from t staged in shared memory, stored coalesced into Y.
// Scheduling: with a single token tile (decode) every CTA owns a contiguous run of tiles;
// otherwise items are dealt round-robin with the token tile varying fastest, so CTAs
// working on the same rows run together and re-read them from L2.
// Every mbarrier wait is bounded (about a second of SM cycles); a wait that gives up sets
// the device error word, the CTA drains what it issued and frees its tensor memory.
#include "tc_common.cuh"

namespace archead {
namespace {

constexpr int kTcThreads = 320;  // warps 0-3 dequant, 4-7 epilogue, 8 producer, 9 MMA
constexpr int kPkBytes = 8192;   // packed block of one 128-row tile (128 columns)

struct TcParams {
  const __half* Hb;  // blocked FP16 H: [token tile][128-column block][NT x 128 image]
  const float* t;    // N x RR
  const uint8_t* nib;
  const uint8_t* code;  // Vpad x G
  const uint16_t* sup;
  const int8_t* Ac;
  const float* sAc;
  const int8_t* Aw;
  const float* sAw;
  float* Y;
  const int32_t* targets;  // fused NLL: target ids (N)
  float2* part;            // fused NLL: (max, sum exp) per (token, vocabulary tile)
  float* tlogit;           // fused NLL: the target's logit per token
  int64_t N, V, D;
  int r_c, r_r, g_shift;
  int n_tok_tiles;
  int64_t n_vtiles;
  unsigned* err;
};

template <int NT>
struct TcCfg {
  static constexpr int SB = NT <= 16 ? 8 : (NT <= 32 ? 4 : 3);  // H ring stages
  static constexpr int SP = NT <= 32 ? 6 : 4;                   // packed ring stages
  static constexpr int HSTAGE = NT * 256;  // bytes of one 128-column H block
  static constexpr int TMEM_COLS = NT <= 64 ? 256 : 512;
  // A-ring stages (64 columns each) in what the two accumulators leave, at most 4
  static constexpr int SA = (TMEM_COLS - 2 * NT) / 64 < 4 ? (TMEM_COLS - 2 * NT) / 64 : 4;
  static_assert(SA >= 2 && 2 * NT + 64 * SA <= TMEM_COLS, "tensor memory budget");
  static_assert(NT % 16 == 0 && NT >= 16 && NT <= 256, "M=128 MMA needs N in 16..256");
};

__host__ __device__ inline size_t round16(size_t x) { return (x + 15) & ~(size_t)15; }

// fused-NLL scratch: a 16-token x 128-row transposed logit chunk plus the tile's targets
template <int NT>
constexpr size_t nll_scratch_bytes() {
  return (size_t)16 * 128 * 4 + (size_t)NT * 4;
}

template <int NT, int MODE>
size_t tc_smem_bytes(int RR, int G) {
  using C = TcCfg<NT>;
  return (size_t)C::SB * C::HSTAGE + (size_t)C::SP * kPkBytes + 2 * round16((size_t)128 * G) +
         round16((size_t)RR * NT * 4) + (MODE ? nll_scratch_bytes<NT>() : 0) + 512;
}

// The k-th work item of this CTA: its tile's first row, its row limit, its token tile.
struct Item {
  int64_t vt, row0, row_end;
  int tt;
};

__device__ __forceinline__ bool get_item(const TcParams& p, int k, Item& it) {
  if (p.n_tok_tiles == 1) {
    const int64_t t0 = p.n_vtiles * blockIdx.x / gridDim.x;
    const int64_t t1 = p.n_vtiles * (blockIdx.x + 1) / gridDim.x;
    it.vt = t0 + k;
    if (it.vt >= t1) return false;
    it.tt = 0;
  } else {
    const int64_t gi = blockIdx.x + (int64_t)k * gridDim.x;
    if (gi >= p.n_vtiles * p.n_tok_tiles) return false;
    it.vt = gi / p.n_tok_tiles;
    it.tt = (int)(gi - it.vt * p.n_tok_tiles);
  }
  it.row0 = it.vt * 128;
  it.row_end = it.row0 + 128 < p.V ? it.row0 + 128 : p.V;
  return true;
}

template <int NT, int CPC, int DQ, int MODE>
__global__ void __launch_bounds__(kTcThreads, 2) residual_tc_kernel(const TcParams p) {
  using C = TcCfg<NT>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int RR = p.r_c + p.r_r;
  const int64_t D = p.D;
  const int nkb = (int)(D / 128);
  const int G = (int)(D >> p.g_shift);
  const int code_bytes = 128 * G;
  unsigned char* Hs = smem;
  unsigned char* pk = Hs + C::SB * C::HSTAGE;
  unsigned char* cds = pk + C::SP * kPkBytes;  // [2][128 x G]
  float* ts = reinterpret_cast<float*>(cds + 2 * round16(code_bytes));  // ts[j * NT + n]
  float* nll_y = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(ts) +
                                          round16((size_t)RR * NT * 4));  // [16][128]
  int32_t* tgt_s = reinterpret_cast<int32_t*>(nll_y + 16 * 128);          // [NT]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(ts) +
                                               round16((size_t)RR * NT * 4) +
                                               (MODE ? nll_scratch_bytes<NT>() : 0));
  uint64_t* b_full = bars;
  uint64_t* b_empty = b_full + C::SB;
  uint64_t* p_full = b_empty + C::SB;
  uint64_t* p_empty = p_full + C::SP;
  uint64_t* c_full = p_empty + C::SP;   // [2]
  uint64_t* c_empty = c_full + 2;       // [2]
  uint64_t* a_full = c_empty + 2;
  uint64_t* a_empty = a_full + C::SA;
  uint64_t* acc_full = a_empty + C::SA;  // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SB; ++s) {
      tc::mbar_init(&b_full[s], 1);
      tc::mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < C::SP; ++s) {
      tc::mbar_init(&p_full[s], 1);
      tc::mbar_init(&p_empty[s], 4);  // one arrival per dequant warp
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&c_full[s], 1);
      tc::mbar_init(&c_empty[s], 4);
      tc::mbar_init(&acc_full[s], 1);
      tc::mbar_init(&acc_empty[s], 128);
    }
    for (int s = 0; s < C::SA; ++s) {
      tc::mbar_init(&a_full[s], 128);
      tc::mbar_init(&a_empty[s], 1);
    }
    tc::mbar_init(mma_done, 1);
    tc::mbar_fence_init();
  }
  if (warp == 9) tc::tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  const uint32_t acol = tbase + 2 * NT;  // A ring after the two accumulators (lane 0)

  if (warp == 8) {
    // ---------------- producers: lane 0 codes + packed blocks, lane 1 H blocks ----------
    // Two independent streams, so the packed prefetch is not held back by the H ring
    // (whose stages free up only as MMAs retire).
    if (lane == 0) {
      int k = 0, np = 0, nc = 0;
      bool ok = true;
      Item it;
      for (int i = 0; ok && get_item(p, i, it); ++i) {
        const int cs = i & 1;
        if (i >= 2 && !tc::mbar_wait(&c_empty[cs], ((i >> 1) - 1) & 1, p.err)) {
          ok = false;
          break;
        }
        tc::fence_proxy_async_smem();  // the stage was read with generic loads
        tc::mbar_arrive_expect_tx(&c_full[cs], (uint32_t)code_bytes);
        tc::bulk_g2s(cds + cs * round16(code_bytes), p.code + it.row0 * G, (uint32_t)code_bytes,
                     &c_full[cs]);
        ++nc;
        const uint8_t* psrc = p.nib + ((it.vt * nkb) << 13);
        for (int kb = 0; kb < nkb; ++kb, ++k) {
          const int sp = k % C::SP;
          if (k >= C::SP && !tc::mbar_wait(&p_empty[sp], ((k / C::SP) - 1) & 1, p.err)) {
            ok = false;
            break;
          }
          tc::fence_proxy_async_smem();  // the stage was read with generic loads
          tc::mbar_arrive_expect_tx(&p_full[sp], kPkBytes);
          tc::bulk_g2s(pk + sp * kPkBytes, psrc + ((int64_t)kb << 13), kPkBytes, &p_full[sp]);
          ++np;
        }
      }
      if (!ok) {  // drain copies still in flight before the CTA exits
        for (int q = np - C::SP < 0 ? 0 : np - C::SP; q < np; ++q)
          tc::mbar_wait(&p_full[q % C::SP], (q / C::SP) & 1, p.err);
        for (int q = nc - 2 < 0 ? 0 : nc - 2; q < nc; ++q)
          tc::mbar_wait(&c_full[q & 1], (q >> 1) & 1, p.err);
      }
    } else if (lane == 1) {
      int k = 0, nb = 0;
      bool ok = true;
      Item it;
      for (int i = 0; ok && get_item(p, i, it); ++i) {
        const unsigned char* hsrc =
            reinterpret_cast<const unsigned char*>(p.Hb) + (int64_t)it.tt * nkb * C::HSTAGE;
        for (int kb = 0; kb < nkb; ++kb, ++k) {
          const int sb = k % C::SB;
          if (k >= C::SB && !tc::mbar_wait(&b_empty[sb], ((k / C::SB) - 1) & 1, p.err)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(&b_full[sb], C::HSTAGE);
          tc::bulk_g2s(Hs + sb * C::HSTAGE, hsrc + (int64_t)kb * C::HSTAGE, C::HSTAGE, &b_full[sb]);
          ++nb;
        }
      }
      if (!ok) {
        for (int q = nb - C::SB < 0 ? 0 : nb - C::SB; q < nb; ++q)
          tc::mbar_wait(&b_full[q % C::SB], (q / C::SB) & 1, p.err);
      }
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_f16_m128(NT);
      int k = 0;
      bool ok = true;
      Item it;
      for (int i = 0; ok && get_item(p, i, it); ++i) {
        const int ab = i & 1;
        if (i >= 2 && !tc::mbar_wait(&acc_empty[ab], ((i >> 1) - 1) & 1, p.err)) break;
        tc::fence_after_sync();
        const uint32_t dcol = tbase + ab * NT;
        for (int kb = 0; kb < nkb; ++kb, ++k) {
          const int sa = k % C::SA, sb = k % C::SB;
          if (!tc::mbar_wait(&a_full[sa], (k / C::SA) & 1, p.err) ||
              !tc::mbar_wait(&b_full[sb], (k / C::SB) & 1, p.err)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t hb = tc::smem_u32(Hs + sb * C::HSTAGE);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            // K step j: 64-column half j / 4 (NT x 128 bytes each), 32-byte offset j % 4
            const uint64_t bd =
                tc::smem_desc_kmajor_sw128(hb + (j >> 2) * NT * 128 + (j & 3) * 32);
            tc::mma_f16_ts(dcol, acol + 64 * sa + 8 * j, bd, idesc, (kb | j) != 0);
          }
          tc::mma_commit(&a_empty[sa]);
          tc::mma_commit(&b_empty[sb]);
        }
        if (ok) tc::mma_commit(&acc_full[ab]);
      }
      tc::mma_commit(mma_done);
      tc::mbar_wait(mma_done, 0, p.err);  // every MMA issued here has retired
    }
  } else if (warp < 4) {
    // ---------------- dequant: thread = tile row = TMEM lane ----------------
    const int tid = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    int k = 0;
    bool ok = true;
    Item it;
    for (int i = 0; ok && get_item(p, i, it); ++i) {
      const int cs = i & 1;
      // warp-uniform outcomes: the tcgen05 stores below are whole-warp instructions
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&c_full[cs], (i >> 1) & 1, p.err))) {
        ok = false;
        break;
      }
      const unsigned char* crow = cds + cs * round16(code_bytes) + tid * G;
      for (int kb = 0; kb < nkb; ++kb, ++k) {
        const int sp = k % C::SP, sa = k % C::SA;
        if (!__all_sync(0xffffffffu, tc::mbar_wait(&p_full[sp], (k / C::SP) & 1, p.err))) {
          ok = false;
          break;
        }
        const unsigned char* src = pk + sp * kPkBytes + tid * 16;
        uint32_t wd[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 u = *reinterpret_cast<const uint4*>(src + c * 128 * 16);
          wd[4 * c + 0] = u.x;
          wd[4 * c + 1] = u.y;
          wd[4 * c + 2] = u.z;
          wd[4 * c + 3] = u.w;
        }
        uint32_t cw[4];
        if (CPC == 1) {
          cw[0] = cw[1] = cw[2] = cw[3] = crow[(kb * 128) >> p.g_shift];
        } else if (CPC == 2) {
          cw[0] = cw[1] = crow[kb * 2];
          cw[2] = cw[3] = crow[kb * 2 + 1];
        } else {
#pragma unroll
          for (int w = 0; w < 4; ++w) cw[w] = crow[kb * 4 + w];
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&p_empty[sp]);
        if (k >= C::SA) {
          if (!__all_sync(0xffffffffu,
                          tc::mbar_wait(&a_empty[sa], ((k / C::SA) - 1) & 1, p.err))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
        }
        const uint32_t ta = acol + 64 * sa + lane_off;
        // window w (32 block columns) = TMEM columns 16w..16w+15: words w, 4+w, 8+w, 12+w
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const __half2 c2 = __half2half2(__ushort2half_rn((unsigned short)cw[w]));
          uint32_t a16[16];
#pragma unroll
          for (int t4 = 0; t4 < 4; ++t4) {
            __half2 pr[4];
            if (DQ == 0) {
              dequant_word(wd[4 * t4 + w], c2, __hmul2(c2, __float2half2_rn(-24.f)), pr);
            } else {
              dequant_word_lite(wd[4 * t4 + w], c2, pr);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) a16[4 * t4 + q] = h2_bits(pr[q]);
          }
          tc::tmem_st16(ta + 16 * w, a16);
        }
        tc::tmem_wait_st();
        tc::fence_before_sync();
        tc::mbar_arrive(&a_full[sa]);
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c_empty[cs]);
    }
  } else if (warp < 8) {
    // ---------------- epilogue: thread = accumulator row = TMEM lane ----------------
    const int e = threadIdx.x - 128;
    const uint32_t lane_off = (uint32_t)(32 * (warp - 4)) << 16;
    int cur_tt = -1;
    Item it;
    for (int i = 0; get_item(p, i, it); ++i) {
      const int ab = i & 1;
      if (it.tt != cur_tt) {  // stage t of this token tile (transposed: ts[j * NT + n])
        asm volatile("bar.sync 1, 128;\n" ::: "memory");
        const int64_t tok0 = (int64_t)it.tt * NT;
        for (int q = e; q < NT * RR; q += 128) {
          const int j = q / NT, n = q - j * NT;
          const int64_t tok = tok0 + n;
          ts[q] = tok < p.N ? __ldg(p.t + tok * RR + j) : 0.f;
        }
        if (MODE == 1)
          for (int q = e; q < NT; q += 128) tgt_s[q] = tok0 + q < p.N ? __ldg(p.targets + tok0 + q) : -1;
        asm volatile("bar.sync 1, 128;\n" ::: "memory");
        cur_tt = it.tt;
      }
      // one outcome for all four epilogue warps: they share named barriers below
      if (!tc::bar_and(1, 128, tc::mbar_wait(&acc_full[ab], (i >> 1) & 1, p.err))) break;
      tc::fence_after_sync();
      const int64_t v = it.row0 + e;
      const bool live = v < it.row_end;
      const int64_t vc = live ? v : it.row0;
      const float S = bf16_bits_to_float(__ldg(p.sup + vc));
      const float sac = p.r_c ? __ldg(p.sAc + vc) : 0.f;
      const float saw = p.r_r ? __ldg(p.sAw + vc) : 0.f;
      const int8_t* arow_c = p.Ac + vc * p.r_c;
      const int8_t* arow_w = p.Aw + vc * p.r_r;
      const int64_t tok0 = (int64_t)it.tt * NT;
#pragma unroll 1
      for (int c = 0; c < NT / 16; ++c) {
        float y[16];
        tc::tmem_ld16(tbase + ab * NT + lane_off + 16 * c, y);
#pragma unroll
        for (int q = 0; q < 16; ++q) y[q] *= S;
#pragma unroll 1
        for (int part = 0; part < 2; ++part) {
          const int rank = part == 0 ? p.r_c : p.r_r;
          if (rank == 0) continue;
          const int8_t* arow = part == 0 ? arow_c : arow_w;
          const float* tcol = ts + (part == 0 ? 0 : p.r_c) * NT + 16 * c;
          float lr[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) lr[q] = 0.f;
          auto acc_j = [&](float aj, int j) {
            const float4* tp = reinterpret_cast<const float4*>(tcol + j * NT);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 tv = tp[q];
              lr[4 * q + 0] = fmaf(aj, tv.x, lr[4 * q + 0]);
              lr[4 * q + 1] = fmaf(aj, tv.y, lr[4 * q + 1]);
              lr[4 * q + 2] = fmaf(aj, tv.z, lr[4 * q + 2]);
              lr[4 * q + 3] = fmaf(aj, tv.w, lr[4 * q + 3]);
            }
          };
          int j = 0;
          if ((rank & 3) == 0 && ((reinterpret_cast<uintptr_t>(arow) & 3) == 0)) {
            // four INT8 factor entries per 32-bit load
            const uint32_t* aw4 = reinterpret_cast<const uint32_t*>(arow);
#pragma unroll 2
            for (; j < rank; j += 4) {
              const uint32_t wv = __ldg(aw4 + (j >> 2));
              acc_j((float)(int8_t)(wv & 0xFF), j);
              acc_j((float)(int8_t)((wv >> 8) & 0xFF), j + 1);
              acc_j((float)(int8_t)((wv >> 16) & 0xFF), j + 2);
              acc_j((float)(int8_t)(wv >> 24), j + 3);
            }
          }
          for (; j < rank; ++j) acc_j((float)__ldg(arow + j), j);
          const float sc = part == 0 ? sac : saw;
#pragma unroll
          for (int q = 0; q < 16; ++q) y[q] = fmaf(sc, lr[q], y[q]);
        }
        if (MODE == 0) {
          if (live) {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int64_t tok = tok0 + 16 * c + q;
              if (tok < p.N) p.Y[tok * p.V + v] = y[q];
            }
          }
        } else {
          // ---- fused NLL: per token of the chunk, (max, sum exp) over the tile's rows ----
          const float NEG_INF = __int_as_float(0xff800000);
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            nll_y[q * 128 + e] = live ? y[q] : NEG_INF;
            const int tg = tgt_s[16 * c + q];
            if (live && tg == v) p.tlogit[tok0 + 16 * c + q] = y[q];
          }
          asm volatile("bar.sync 1, 128;\n" ::: "memory");
          // thread e: token q = e / 8 of the chunk, rows 16 * (e % 8) .. +15
          const int q = e >> 3, seg = e & 7;
          const float* yr = nll_y + q * 128 + 16 * seg;
          float m = NEG_INF;
#pragma unroll
          for (int i = 0; i < 16; ++i) m = fmaxf(m, yr[i]);
          float sm = 0.f;
          if (m != NEG_INF) {
#pragma unroll
            for (int i = 0; i < 16; ++i) sm += __expf(yr[i] - m);
          }
#pragma unroll
          for (int o = 1; o < 8; o <<= 1) {  // combine the 8 segments of the token
            const float mo = __shfl_xor_sync(0xffffffffu, m, o);
            const float so = __shfl_xor_sync(0xffffffffu, sm, o);
            const float mn = fmaxf(m, mo);
            sm = (m == NEG_INF ? 0.f : sm * __expf(m - mn)) + (mo == NEG_INF ? 0.f : so * __expf(mo - mn));
            m = mn;
          }
          const int64_t tok = tok0 + 16 * c + q;
          if (seg == 0 && tok < p.N) p.part[tok * p.n_vtiles + it.vt] = make_float2(m, sm);
          asm volatile("bar.sync 1, 128;\n" ::: "memory");
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&acc_empty[ab]);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// FP16 copy of H in the image the MMA's B operand reads: for token tile tt of NT rows and
// 128-column block kb, a contiguous NT x 128 block made of two 64-column halves; in half h
// the 16-byte piece (token n, columns 64h + 8c .. +7) sits at h * NT * 128 + n * 128 +
// (c ^ (n % 8)) * 16 bytes (K-major, 128-byte swizzle).  Rows >= N are zero.  Non-finite
// or out-of-range FP16 values set kErrRangeH.
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
    const int64_t kb = kc >> 4, half = (kc >> 3) & 1, c = kc & 7;
    const int64_t off = (tt * nkb + kb) * (int64_t)nt * 128 + half * (int64_t)nt * 64 + nn * 64 +
                        ((c ^ (nn & 7)) * 8);
    *reinterpret_cast<uint4*>(Hb + off) = out;
  }
  if (bad) atomicOr(err, kErrRangeH);
}

template <int NT, int CPC, int DQ, int MODE>
cudaError_t launch_tc_cfg(const TcParams& p, cudaStream_t st) {
  const int RR = p.r_c + p.r_r;
  const size_t smem = tc_smem_bytes<NT, MODE>(RR, (int)(p.D >> p.g_shift));
  auto kern = residual_tc_kernel<NT, CPC, DQ, MODE>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, smem_sm = 0, regs_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) !=
          cudaSuccess ||
      (e = cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev)) !=
          cudaSuccess)
    return e;
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
  // resident CTAs per SM: registers (allocated per warp in units of 256), shared memory
  // (plus the 1 KB the driver reserves per CTA), warps, and tensor-memory columns
  const int warps = kTcThreads / 32;
  const int regs_warp = (fa.numRegs * 32 + 255) / 256 * 256;
  int occ = regs_sm / (regs_warp * warps);
  const int by_smem = smem_sm / (int)(smem + fa.sharedSizeBytes + 1024);
  if (by_smem < occ) occ = by_smem;
  if (64 / warps < occ) occ = 64 / warps;
  if (512 / TcCfg<NT>::TMEM_COLS < occ) occ = 512 / TcCfg<NT>::TMEM_COLS;
  if (occ < 1) occ = 1;
  int64_t items = p.n_vtiles * p.n_tok_tiles;
  int64_t grid = (int64_t)sms * occ;
  if (grid > items) grid = items;
  kern<<<(unsigned)grid, kTcThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <int NT, int MODE>
cudaError_t launch_tc_nt(const TcParams& p, int g, cudaStream_t st) {
  if (g == 32) return launch_tc_cfg<NT, 4, 1, MODE>(p, st);
  if (g == 64) return launch_tc_cfg<NT, 2, 1, MODE>(p, st);
  return launch_tc_cfg<NT, 1, 1, MODE>(p, st);
}

template <int MODE>
cudaError_t launch_tc_mode(const TcParams& p, int nt, int g, cudaStream_t st) {
  switch (nt) {
    case 16: return launch_tc_nt<16, MODE>(p, g, st);
    case 32: return launch_tc_nt<32, MODE>(p, g, st);
    case 64: return launch_tc_nt<64, MODE>(p, g, st);
    default: return launch_tc_nt<128, MODE>(p, g, st);
  }
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
                               const Shapes& s, float* Y, const int32_t* targets, float2* part,
                               float* tlogit, unsigned* err, cudaStream_t st, int* launches) {
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
  p.err = err;
  const int nt = tc_token_tile(s.N, s.r_c + s.r_r);
  p.n_tok_tiles = (int)((s.N + nt - 1) / nt);
  p.n_vtiles = (s.V + 127) / 128;
  cudaError_t e = Y ? launch_tc_mode<0>(p, nt, s.g, st) : launch_tc_mode<1>(p, nt, s.g, st);
  ++*launches;
  return e;
}

}  // namespace archead
