// Logit contraction on the 5th-generation tensor cores (tcgen05, TMEM accumulators).
//
//   Y[n, v] = S_v sum_d h[n, d] q[v, d] c[v, d / g]  +  sum_j a[v, j] t[n, j]   (ARCHead Sec. 3)
//
// with a = [Q8(A_c) | Q8(A_w)] (row-scaled INT8) and t = H [Q8(B_c) | Q8(B_w)]^T.  Both sums
// run on the tensor cores into ONE FP32 accumulator per (row, token), scaled by a per-row
// S'_v = S_v 2^k_v:
//   * residual K columns: A = q c 2^-k (exact in FP16 for k <= 24), B = fp16(h);
//   * rank K columns (4 per factor index j): A = (x1, x1, x2, x2), B = (t1, t2, t1, t2),
//     where x = a / S' and t are each split into an FP16 hi piece and an FP16 remainder, so
//     x1 t1 + x1 t2 + x2 t1 + x2 t2 carries about 22 significant bits of a t / S';
//   * the epilogue writes S'_v times the accumulator.
// k_v is chosen from the row's scales alone: every factor entry obeys |a| <= 128 max(sAc,
// sAw), and k puts that bound between 2^12 and 2^14 after division by S', far inside FP16.
//
// Persistent, warp-specialised kernel, two CTAs per SM.  A work item is one 128-row
// vocabulary tile for one tile of NT tokens (NT = 16..128), or a K range of it:
//  * warp 8 (one thread) feeds the packed ring with bulk copies (TMA engine, no tensor
//    map, no multicast): the tile's group-scale codes once per item, then its 8 KB
//    packed-nibble block per 128 columns (one contiguous region in the tiled device
//    layout); warp 10 (one thread) feeds the B ring with the token tile's FP16 blocks
//    (pre-arranged by the prologue as the 128-byte-swizzled K-major image the MMA reads).
//    Each waits (blocking) for the slot it refills, so neither stream waits behind the
//    other and neither takes issue slots from the dequant warps while it waits;
//  * warps 0-3 (dequant): one vocabulary row per thread (= one TMEM lane).  A thread reads
//    its row's four 16-byte chunks of a block (conflict free: chunk i of row s sits at
//    (i * 128 + s) * 16), dequantises them to exact FP16 q c 2^-k, and after the residual
//    blocks converts its row's factor entries into the rank blocks; it stores both with
//    tcgen05.st into an A ring of 2-3 stages in tensor memory (128 x 128 FP16 = 64
//    columns per stage);
//  * warp 9 (the whole warp, one elected lane issues): tcgen05.mma kind::f16, A from
//    tensor memory, B from shared memory, K=16 steps, into an M=128 x N=NT FP32
//    accumulator (two of them below NT = 128, so the next item's MMAs overlap the
//    previous item's epilogue);
//  * warps 4-7 (epilogue): tcgen05.ld of an accumulator row, times S'_v, stored into Y, or
//    reduced on chip into split-vocabulary log-sum-exp partials (fused NLL).
// Scheduling: with a single token tile (decode) the (tile, K block) units are split evenly
// over the CTAs and a tile at the edge of two ranges is finished from two partial
// accumulators; otherwise the CTAs take items in order (the token tile varying fastest
// inside L2-sized bands) from a work counter: the packed producer claims them two items
// ahead of its stream and hands the indices to the other roles through a small queue in
// shared memory, so all CTAs stay within a few items of one another and the readers of a
// vocabulary tile find its packed blocks in L2.
// Every mbarrier wait is bounded (about a second of SM cycles); a wait that gives up sets
// the device error word, the CTA drains what it issued and frees its tensor memory.
#include "tc_common.cuh"

namespace archead {
namespace {

constexpr int kTcThreads = 352;  // warps 0-3 dequant, 4-7 epilogue, 8 and 10 producers, 9 MMA
constexpr int kPkBytes = 8192;   // packed block of one 128-row tile (128 columns)
constexpr int kMaxSB = 8;        // deepest B ring
constexpr int kMaxSP = 8;        // deepest packed ring
constexpr int kItemQ = 8;        // item queue slots (dynamic order)
constexpr int kItemAhead = 2;    // items the packed producer claims ahead of its stream
constexpr int kItemUsers = 10;   // releases per item: B producer, MMA warp, 4 dequant, 4 epilogue

struct TcParams {
  const __half* Hb;  // B image: [token tile][nkb + nrb blocks][NT x 128]
  const float* tsc;  // N token scales 2^e_n (the image holds H 2^-e_n)
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
  int nrb;         // rank blocks after the residual blocks
  int rank_steps;  // K=16 steps holding rank columns: ceil(4 (r_c + r_r) / 16)
  int a_words;     // factor rows readable as aligned 32-bit words
  int sb;          // B ring stages (<= kMaxSB)
  int spk;         // packed ring stages (<= kMaxSP)
  int n_tok_tiles;
  int tt_band;  // token tiles per band (their B image stays in L2 while the head streams)
  int64_t n_vtiles;
  // One token tile: the (tile, K block) units are split evenly over the CTAs, so a tile
  // at the edge of a CTA's range is shared with the neighbouring CTA (its "head" blocks
  // in one, its "tail" blocks in the next).  Each part's raw accumulator goes to scratch
  // ([CTA][slot 0: first item, 1: last item][NT][128] FP32); the part that arrives second
  // at the tile's counter (zeroed by the prologue) adds the two and finishes the tile.
  int split;
  // Several token tiles: the items are taken in order from a work counter (counters[0],
  // zeroed by the prologue) instead of a fixed round-robin, so all CTAs stay within a few
  // items of one another and the readers of a vocabulary tile share its reads through L2.
  int dyn;
  float* scratch;
  unsigned* counters;
  unsigned* err;
};

template <int NT>
struct TcCfg {
  static constexpr int HSTAGE = NT * 256;      // bytes of one 128-column B block
  // Two CTAs per SM (256 TMEM columns each) for every tile: a single MMA issuer per SM
  // sustains only about one 8-MMA stage per ~950 cycles (stage handshakes ride on commit
  // and mbarrier latencies), two issuers fill each other's gaps.  The 128-token tile keeps
  // one accumulator, which the epilogue frees once its last 32-column batch is in
  // registers (two A stages fit beside it); smaller tiles double-buffer the accumulator,
  // so the next item's MMAs never wait for the epilogue, and keep two (NT = 64) or three
  // A stages.  An A stage is reused only after the MMAs reading it have completed (about
  // a thousand cycles after their issue); at these depths the dequant warps, not the
  // ring, set the stage rate.
  static constexpr int TMEM_COLS = 256;
  static constexpr int NACC = NT == 128 ? 1 : 2;
  // A-ring stages (64 columns each) in what the accumulators leave, at most 4
  static constexpr int SA =
      (TMEM_COLS - NACC * NT) / 64 < 4 ? (TMEM_COLS - NACC * NT) / 64 : 4;
  static_assert(SA >= 2 && NACC * NT + 64 * SA <= TMEM_COLS, "tensor memory budget");
  static_assert(NT % 16 == 0 && NT >= 16 && NT <= 256, "M=128 MMA needs N in 16..256");
};

__host__ __device__ inline size_t round16(size_t x) { return (x + 15) & ~(size_t)15; }

// fused-NLL scratch: a 16-token x 128-row transposed logit chunk plus the tile's targets
template <int NT>
constexpr size_t nll_scratch_bytes() {
  return (size_t)16 * 128 * 4 + (size_t)NT * 4;
}

template <int NT>
size_t tc_smem_bytes(int sb, int sp, int G, bool nll) {
  using C = TcCfg<NT>;
  return (size_t)sb * C::HSTAGE + (size_t)sp * kPkBytes + 2 * round16((size_t)128 * G) +
         (nll ? nll_scratch_bytes<NT>() : 0) + (size_t)NT * 4 + 1024;
}

// The k-th work item of this CTA: its tile's first row, its row limit, its token tile.
struct Item {
  int64_t vt, row0, row_end;
  int tt;
  int kb0, kb1;  // the item's K blocks [kb0, kb1) of the tile's nkb + nrb
  int part;      // 0: whole tile; 1: head part (blocks from 0); 2: tail part (to the end)
};

// Item gi of the several-token-tile order: bands of tt_band token tiles; inside a band the
// token tile varies fastest, so CTAs reading the same vocabulary rows run together and the
// band's B image is reused from L2 across all vocabulary tiles.  False past the last item.
__device__ __forceinline__ bool item_of(const TcParams& p, int64_t gi, Item& it) {
  if (gi >= p.n_vtiles * p.n_tok_tiles) return false;
  const int64_t band_items = p.n_vtiles * p.tt_band;
  const int64_t band = gi / band_items;
  const int64_t local = gi - band * band_items;
  const int64_t tt0 = band * p.tt_band;
  const int64_t nb = p.n_tok_tiles - tt0 < p.tt_band ? p.n_tok_tiles - tt0 : p.tt_band;
  it.vt = local / nb;
  it.tt = (int)(tt0 + (local - it.vt * nb));
  it.kb0 = 0;
  it.kb1 = (int)(p.D >> 7) + p.nrb;
  it.part = 0;
  it.row0 = it.vt * 128;
  it.row_end = it.row0 + 128 < p.V ? it.row0 + 128 : p.V;
  return true;
}

__device__ __forceinline__ bool get_item(const TcParams& p, int k, Item& it) {
  const int nkbt = (int)(p.D >> 7) + p.nrb;
  it.kb0 = 0;
  it.kb1 = nkbt;
  it.part = 0;
  if (p.split) {
    // units u = tile * nkbt + block, [u0, u1) per CTA; every range spans at least one
    // tile (the grid has at most one CTA per tile), so a tile has at most two parts
    const int64_t U = p.n_vtiles * nkbt;
    const int64_t u0 = U * blockIdx.x / gridDim.x;
    const int64_t u1 = U * (blockIdx.x + 1) / gridDim.x;
    it.vt = u0 / nkbt + k;
    const int64_t ts = it.vt * nkbt;
    if (ts >= u1) return false;
    it.kb0 = u0 > ts ? (int)(u0 - ts) : 0;
    it.kb1 = u1 < ts + nkbt ? (int)(u1 - ts) : nkbt;
    it.part = it.kb0 > 0 ? 2 : (it.kb1 < nkbt ? 1 : 0);
    it.tt = 0;
  } else if (p.n_tok_tiles == 1) {
    const int64_t t0 = p.n_vtiles * blockIdx.x / gridDim.x;
    const int64_t t1 = p.n_vtiles * (blockIdx.x + 1) / gridDim.x;
    it.vt = t0 + k;
    if (it.vt >= t1) return false;
    it.tt = 0;
  } else {
    if (!item_of(p, blockIdx.x + (int64_t)k * gridDim.x, it)) return false;
  }
  it.row0 = it.vt * 128;
  it.row_end = it.row0 + 128 < p.V ? it.row0 + 128 : p.V;
  return true;
}

// The k-th item of this CTA.  The fixed orders come from get_item; the dynamic order from
// the item queue that the packed producer fills: the caller waits for slot k's phase, reads
// the item index, and its warp releases the slot (one arrival per warp, by lane 0 after
// all its lanes have read; `solo` for a single-thread role).
struct ItemQueue {
  const int64_t* ids;
  uint64_t* full;
  uint64_t* empty;
};
__device__ __forceinline__ bool next_item(const TcParams& p, const ItemQueue& q, int64_t k,
                                          Item& it, bool& ok, bool solo) {
  if (!p.dyn) return get_item(p, (int)k, it);
  if (!ok) return false;  // warp-uniform for warp callers: only set from warp-wide outcomes
  const int slot = (int)(k % kItemQ);
  bool got = tc::mbar_wait(&q.full[slot], (uint32_t)(k / kItemQ) & 1u, p.err);
  if (!solo) got = __all_sync(0xffffffffu, got);  // the lanes agree before __syncwarp below
  if (!got) {
    ok = false;
    return false;
  }
  const int64_t gi = *reinterpret_cast<const volatile int64_t*>(q.ids + slot);
  if (solo) {
    tc::mbar_arrive(&q.empty[slot]);
  } else {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) tc::mbar_arrive(&q.empty[slot]);
  }
  return item_of(p, gi, it);
}

// The row scales of vocabulary row v (clamped into range; rows past V only pad a tile).
struct RowIn {
  float S, sac, saw;
};
__device__ __forceinline__ RowIn load_row(const TcParams& p, int64_t v) {
  const int64_t vc = v < p.V ? v : p.V - 1;
  RowIn r;
  r.S = bf16_bits_to_float(__ldg(p.sup + vc));
  r.sac = p.r_c ? __ldg(p.sAc + vc) : 0.f;
  r.saw = p.r_r ? __ldg(p.sAw + vc) : 0.f;
  return r;
}

// Accumulator scale S' = S 2^k of a row and the factor 2^-k applied to its group codes
// (0 when S = 0: the residual row is zero and is dropped).  With M = 128 max(|sAc|, |sAw|)
// bounding every factor entry, k = ilogb(M) - ilogb(S) - 13 puts M / S' in (2^12, 2^14);
// k is clamped to [-3, 40]: the dequant's fused multiply-add takes -24 c 2^-k as an FP16
// operand, and 24 * 255 * 2^3 = 48960 stays finite (a larger k only shrinks M / S'); q c
// 2^-k is exact for k <= 24, and below that the residual is under 2^-30 of the factor
// terms.
struct RowScale {
  float sp, cs;
};
__device__ __forceinline__ RowScale row_scale(const RowIn& in) {
  const float M = 128.f * fmaxf(fabsf(in.sac), fabsf(in.saw));
  RowScale r;
  if (in.S != 0.f) {
    int k = 0;
    if (M > 0.f) {
      k = ilogbf(M) - ilogbf(in.S) - 13;
      k = k < -3 ? -3 : (k > 40 ? 40 : k);
    }
    r.sp = ldexpf(in.S, k);
    r.cs = ldexpf(1.f, -k);
  } else {
    r.sp = M > 0.f ? ldexpf(1.f, ilogbf(M) - 13) : 1.f;
    r.cs = 0.f;
  }
  return r;
}

// Four INT8 factor entries j .. j+3 of row v in the concatenation [A_c | A_w] (zeros past
// r_c + r_r).  With a_words the four never straddle the two factors (r_c % 4 == 0).
__device__ __forceinline__ uint32_t factor_word(const TcParams& p, int64_t v, int j) {
  const int RR = p.r_c + p.r_r;
  if (p.a_words) {
    if (j < p.r_c) return __ldg(reinterpret_cast<const uint32_t*>(p.Ac + v * p.r_c + j));
    if (j < RR) return __ldg(reinterpret_cast<const uint32_t*>(p.Aw + v * p.r_r + (j - p.r_c)));
    return 0u;
  }
  uint32_t w = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int jj = j + u;
    int8_t b = 0;
    if (jj < p.r_c) b = __ldg(p.Ac + v * p.r_c + jj);
    else if (jj < RR) b = __ldg(p.Aw + v * p.r_r + (jj - p.r_c));
    w |= (uint32_t)(uint8_t)b << (8 * u);
  }
  return w;
}

__device__ __forceinline__ void prefetch_l2(const void* ptr) {
  asm volatile("prefetch.global.L2 [%0];\n" ::"l"(ptr));
}

template <int NT, int CPC, int MODE>
__global__ void __launch_bounds__(kTcThreads, 2) residual_tc_kernel(const TcParams p) {
  using C = TcCfg<NT>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int64_t D = p.D;
  const int nkb = (int)(D / 128);
  const int nkbt = nkb + p.nrb;  // B blocks per item
  const int G = (int)(D >> p.g_shift);
  const int code_bytes = 128 * G;
  const int SB = p.sb;
  unsigned char* Hs = smem;
  unsigned char* pk = Hs + SB * C::HSTAGE;
  const int SPK = p.spk;
  unsigned char* cds = pk + SPK * kPkBytes;  // [2][128 x G]
  unsigned char* after_codes = cds + 2 * round16(code_bytes);
  float* nll_y = reinterpret_cast<float*>(after_codes);  // [16][128]
  int32_t* tgt_s = reinterpret_cast<int32_t*>(nll_y + 16 * 128);  // [NT]
  float* tsc_s = reinterpret_cast<float*>(after_codes + (MODE ? nll_scratch_bytes<NT>() : 0));
  uint64_t* bars = reinterpret_cast<uint64_t*>(tsc_s + NT);  // tsc_s: [NT] token scales
  uint64_t* b_full = bars;
  uint64_t* b_empty = b_full + kMaxSB;
  uint64_t* p_full = b_empty + kMaxSB;
  uint64_t* p_empty = p_full + kMaxSP;
  uint64_t* c_full = p_empty + kMaxSP;  // [2]
  uint64_t* c_empty = c_full + 2;       // [2]
  uint64_t* a_full = c_empty + 2;
  uint64_t* a_empty = a_full + C::SA;
  uint64_t* acc_full = a_empty + C::SA;  // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint64_t* item_full = mma_done + 1;        // [kItemQ]
  uint64_t* item_empty = item_full + kItemQ;  // [kItemQ]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(item_empty + kItemQ);
  int* ep_flag = reinterpret_cast<int*>(tmem_slot + 1);  // epilogue: a tile counter's value
  int64_t* item_ids = reinterpret_cast<int64_t*>(tmem_slot + 2);  // [kItemQ]
  const ItemQueue iq = {item_ids, item_full, item_empty};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SB; ++s) {
      tc::mbar_init(&b_full[s], 1);
      tc::mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < SPK; ++s) {
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
    for (int s = 0; s < kItemQ; ++s) {
      tc::mbar_init(&item_full[s], 1);
      tc::mbar_init(&item_empty[s], kItemUsers);
    }
    tc::mbar_fence_init();
  }
  if (warp == 9) tc::tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  const uint32_t acol = tbase + C::NACC * NT;  // A ring after the accumulators (lane 0)

  if (warp == 8) {
    // ---------------- packed producer (one thread) ----------------
    // Each item's group codes, then its packed blocks, each copy as soon as its slot is
    // released (blocking waits: the thread sleeps instead of taking issue slots from the
    // dequant warps).  Ring slots and phases advance incrementally and the source address
    // by a constant stride: the thread is on the critical path of the pipeline.  A wait
    // that gives up drains the copies in flight.
    if (lane == 0) {
      bool ok = true;
      // dynamic order: claim items from the work counter (zeroed by the prologue kernel,
      // hence the dependency wait) kItemAhead ahead of the stream, into the item queue
      int64_t claimed = 0;
      bool more = true;
      const int64_t total = p.n_vtiles * p.n_tok_tiles;
      if (p.dyn) grid_dependency_wait();
      auto claim_to = [&](int64_t upto) {
        while (ok && more && claimed <= upto) {
          const int slot = (int)(claimed % kItemQ);
          if (claimed >= kItemQ &&
              !tc::mbar_wait(&item_empty[slot], (uint32_t)((claimed / kItemQ) - 1) & 1u, p.err)) {
            ok = false;
            break;
          }
          const int64_t gi = (int64_t)atomicAdd(p.counters, 1u);
          item_ids[slot] = gi;
          tc::mbar_arrive(&item_full[slot]);  // releases the index to the waiting roles
          ++claimed;
          if (gi >= total) more = false;
        }
      };
      auto p_next = [&](int64_t k, Item& it) -> bool {
        if (!p.dyn) return get_item(p, (int)k, it);
        claim_to(k + kItemAhead);
        if (!ok || k >= claimed) return false;
        return item_of(p, item_ids[k % kItemQ], it);
      };
      Item pit;
      bool p_have = p_next(0, pit);
      int ip = 0, np = 0, nc = 0, ps = 0, cs = 0;
      uint32_t pph = 0, cph = 0;  // phase parities of the next refill of slot ps / cs
      while (ok && p_have) {
        if (nc >= 2 && !tc::mbar_wait(&c_empty[cs], cph ^ 1u, p.err)) {
          ok = false;
          break;
        }
        tc::fence_proxy_async_smem();  // the slot was read with generic loads
        tc::mbar_arrive_expect_tx(&c_full[cs], (uint32_t)code_bytes);
        tc::bulk_g2s(cds + cs * round16(code_bytes), p.code + pit.row0 * G,
                     (uint32_t)code_bytes, &c_full[cs]);
        ++nc;
        if (++cs == 2) {
          cs = 0;
          cph ^= 1u;
        }
        const int pk1 = pit.kb1 < nkb ? pit.kb1 : nkb;
        const uint8_t* psrc = p.nib + ((pit.vt * nkb + pit.kb0) << 13);
        for (int kb = pit.kb0; kb < pk1; ++kb) {
          if (np >= SPK && !tc::mbar_wait(&p_empty[ps], pph ^ 1u, p.err)) {
            ok = false;
            break;
          }
          tc::fence_proxy_async_smem();  // the stage was read with generic loads
          tc::mbar_arrive_expect_tx(&p_full[ps], kPkBytes);
          tc::bulk_g2s(pk + ps * kPkBytes, psrc, kPkBytes, &p_full[ps]);
          psrc += kPkBytes;
          ++np;
          if (++ps == SPK) {
            ps = 0;
            pph ^= 1u;
          }
        }
        p_have = p_next(++ip, pit);
      }
      if (!ok) {  // drain copies still in flight before the CTA exits
        for (int q = np - SPK < 0 ? 0 : np - SPK; q < np; ++q)
          tc::mbar_wait(&p_full[q % SPK], (q / SPK) & 1, p.err);
        for (int q = nc - 2 < 0 ? 0 : nc - 2; q < nc; ++q)
          tc::mbar_wait(&c_full[q & 1], (q >> 1) & 1, p.err);
      }
    }
  } else if (warp == 10) {
    // ---------------- B producer (one thread) ----------------
    // The token tile's image blocks, one per stage, each as soon as the MMAs that read its
    // slot have completed.  The image comes from the prologue kernels (this kernel is a
    // programmatic dependent launch), so the stream starts after the dependency wait.
    if (lane == 0) {
      grid_dependency_wait();
      Item hit;
      bool ok = true;
      bool h_have = next_item(p, iq, 0, hit, ok, true);
      int ih = 0, nb = 0, hs = 0;
      uint32_t hph = 0;
      while (ok && h_have) {
        const unsigned char* hsrc = reinterpret_cast<const unsigned char*>(p.Hb) +
                                    ((int64_t)hit.tt * nkbt + hit.kb0) * C::HSTAGE;
        for (int kb = hit.kb0; kb < hit.kb1; ++kb) {
          if (nb >= SB && !tc::mbar_wait(&b_empty[hs], hph ^ 1u, p.err)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(&b_full[hs], C::HSTAGE);
          tc::bulk_g2s(Hs + hs * C::HSTAGE, hsrc, C::HSTAGE, &b_full[hs]);
          hsrc += C::HSTAGE;
          ++nb;
          if (++hs == SB) {
            hs = 0;
            hph ^= 1u;
          }
        }
        h_have = next_item(p, iq, ++ih, hit, ok, true);
      }
      if (!ok) {
        for (int q = nb - SB < 0 ? 0 : nb - SB; q < nb; ++q)
          tc::mbar_wait(&b_full[q % SB], (q / SB) & 1, p.err);
      }
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer: the whole warp, one elected lane issues ----------------
    // The issuing thread is on the critical path of the stage ring, so its stream is kept
    // short: ring slots and phases advance incrementally (no division), the B descriptor
    // of a stage is one add to a base descriptor (start address field in 16-byte units;
    // shared-memory addresses stay below 2^18, so the field never carries), the K steps of
    // a residual block are unrolled with constant offsets, and the whole warp runs the
    // loop converged so those values stay warp-uniform; one elected lane issues the MMAs
    // and commits.
    {
      const uint32_t idesc = tc::idesc_f16_m128(NT);
      const uint64_t bdesc0 = tc::smem_desc_kmajor_sw128(tc::smem_u32(Hs));
      int sa = 0, sb = 0;
      uint32_t pa = 0, pb = 0;
      bool ok = true;
      Item it;
      for (int i = 0; ok && __all_sync(0xffffffffu, next_item(p, iq, i, it, ok, false)); ++i) {
        const int ab = i % C::NACC, use = i / C::NACC;
        if (i >= C::NACC &&
            !__all_sync(0xffffffffu, tc::mbar_wait(&acc_empty[ab], (use - 1) & 1, p.err)))
          break;
        tc::fence_after_sync();
        const uint32_t dcol = tbase + ab * NT;
        for (int kb = it.kb0; kb < it.kb1; ++kb) {
          const bool a_rdy = tc::mbar_try_wait(&a_full[sa], pa);
          const bool b_rdy = tc::mbar_try_wait(&b_full[sb], pb);
          if (!__all_sync(0xffffffffu, (a_rdy && b_rdy) ||
                                           (tc::mbar_wait(&a_full[sa], pa, p.err) &&
                                            tc::mbar_wait(&b_full[sb], pb, p.err)))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          // K step j: 64-column half j / 4 (NT x 128 bytes each), 32-byte offset j % 4
          const uint64_t bd = bdesc0 + (uint64_t)((sb * C::HSTAGE) >> 4);
          const uint32_t ad = acol + 64 * sa;
          if (tc::elect_one()) {
            if (kb < nkb) {
#pragma unroll
              for (int j = 0; j < 8; ++j)
                tc::mma_f16_ts(dcol, ad + 8 * j,
                               bd + (((j >> 2) * NT * 128 + (j & 3) * 32) >> 4), idesc,
                               (kb != it.kb0) | (j != 0));
            } else {
              // rank blocks: the K steps that hold factor columns
              const int steps = min(8, p.rank_steps - 8 * (kb - nkb));
#pragma unroll
              for (int j = 0; j < 8; ++j)
                if (j < steps)
                  tc::mma_f16_ts(dcol, ad + 8 * j,
                                 bd + (((j >> 2) * NT * 128 + (j & 3) * 32) >> 4), idesc,
                                 (kb != it.kb0) | (j != 0));
            }
            tc::mma_commit(&a_empty[sa]);
            tc::mma_commit(&b_empty[sb]);
          }
          __syncwarp();
          if (++sa == C::SA) {
            sa = 0;
            pa ^= 1u;
          }
          if (++sb == SB) {
            sb = 0;
            pb ^= 1u;
          }
        }
        if (ok && tc::elect_one()) tc::mma_commit(&acc_full[ab]);
        __syncwarp();
      }
      if (tc::elect_one()) {
        tc::mma_commit(mma_done);
        tc::mbar_wait(mma_done, 0, p.err);  // every MMA issued here has retired
      }
      __syncwarp();
    }
  } else if (warp < 4) {
    // ---------------- dequant: thread = tile row = TMEM lane ----------------
    const int tid = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    int k = 0;   // A-ring sequence: residual and rank blocks
    // packed-ring position of the next residual block (the ring carries residual blocks
    // only): slot and phase parity, kept incrementally
    int sp = 0;
    uint32_t spar = 0;
    bool p_ready = false, a_ready = false;  // the next stage's barriers, probed early
    bool ok = true;
    Item it;
    bool have = __all_sync(0xffffffffu, next_item(p, iq, 0, it, ok, false));
    RowIn rin = {0.f, 0.f, 0.f};
    if (have) rin = load_row(p, it.row0 + tid);
    for (int i = 0; ok && have; ++i) {
      // the next item's row scales load while this one runs
      Item nx;
      const bool have_nx = __all_sync(0xffffffffu, next_item(p, iq, i + 1, nx, ok, false));
      RowIn rnx = rin;
      if (have_nx) rnx = load_row(p, nx.row0 + tid);
      const int64_t v = it.row0 + tid;
      const bool live = v < it.row_end;
      const RowScale rs = row_scale(rin);
      if (live && p.nrb) {  // the factor rows are read after the residual blocks
        if (p.r_c) prefetch_l2(p.Ac + v * p.r_c);
        if (p.r_r) prefetch_l2(p.Aw + v * p.r_r);
      }
      const int cs = i & 1;
      // warp-uniform outcomes: the tcgen05 stores below are whole-warp instructions
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&c_full[cs], (i >> 1) & 1, p.err))) {
        ok = false;
        break;
      }
      const unsigned char* crow = cds + cs * round16(code_bytes) + tid * G;
      const int kr1 = it.kb1 < nkb ? it.kb1 : nkb;
      for (int kb = it.kb0; kb < kr1; ++kb, ++k) {
        const int sa = k % C::SA;
        if (!__all_sync(0xffffffffu, p_ready) &&
            !__all_sync(0xffffffffu, tc::mbar_wait(&p_full[sp], spar, p.err))) {
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
        if (++sp == SPK) {
          sp = 0;
          spar ^= 1u;
        }
        if (k >= C::SA) {
          if (!__all_sync(0xffffffffu, a_ready) &&
              !__all_sync(0xffffffffu,
                          tc::mbar_wait(&a_empty[sa], ((k / C::SA) - 1) & 1, p.err))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
        }
        // The next stage's barriers are probed now and their answers used only after this
        // stage's arithmetic, which hides the shared-memory round trip of the probe; a
        // phase seen complete stays complete until this thread releases the slot.
        p_ready = tc::mbar_test(&p_full[sp], spar);
        a_ready = k + 1 < C::SA || tc::mbar_test(&a_empty[(k + 1) % C::SA], (((k + 1) / C::SA) - 1) & 1);
        const uint32_t ta = acol + 64 * sa + lane_off;
        // window w (32 block columns) = TMEM columns 16w..16w+15: words w, 4+w, 8+w, 12+w
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          // c 2^-k is exact in FP16 (8 significant bits, k <= 24)
          const __half2 c2 = __float2half2_rn((float)cw[w] * rs.cs);
          const __half2 nc24 = __hmul2(c2, __float2half2_rn(-24.f));  // exact: 3 c 2^(3-k)
          uint32_t a16[16];
#pragma unroll
          for (int t4 = 0; t4 < 4; ++t4) {
            __half2 pr[4];
            dequant_word(wd[4 * t4 + w], c2, nc24, pr);
#pragma unroll
            for (int q = 0; q < 4; ++q) a16[4 * t4 + q] = h2_bits(pr[q]);
          }
          tc::tmem_st16(ta + 16 * w, a16);
        }
        tc::tmem_wait_st();
        tc::fence_before_sync();
        tc::mbar_arrive(&a_full[sa]);
      }
      a_ready = false;  // probed for the next A stage, which the rank blocks wait for themselves
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c_empty[cs]);
      // rank blocks: factor index j = 32 rb + i takes TMEM columns 2i (x1, x1) and
      // 2i + 1 (x2, x2), x = fl32(A[v, j] s_v) / S' split into FP16 hi and remainder
      const float rcp = 1.f / rs.sp;
      const int rb1 = it.kb1 - nkb;
      for (int rb = it.kb0 > nkb ? it.kb0 - nkb : 0; ok && rb < rb1; ++rb, ++k) {
        const int sa = k % C::SA;
        uint32_t fw[8];
#pragma unroll
        for (int w = 0; w < 8; ++w) fw[w] = live ? factor_word(p, v, 32 * rb + 4 * w) : 0u;
        if (k >= C::SA) {
          if (!__all_sync(0xffffffffu,
                          tc::mbar_wait(&a_empty[sa], ((k / C::SA) - 1) & 1, p.err))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
        }
        const uint32_t ta = acol + 64 * sa + lane_off;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t a16[16];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = 32 * rb + 8 * q4 + u;
            const int8_t e = (int8_t)((fw[2 * q4 + (u >> 2)] >> (8 * (u & 3))) & 0xFFu);
            const float x = __fmul_rn((float)e, j < p.r_c ? rin.sac : rin.saw) * rcp;
            const __half x1 = __float2half_rn(x);
            const __half x2 = __float2half_rn(x - __half2float(x1));
            a16[2 * u] = h2_bits(__half2half2(x1));
            a16[2 * u + 1] = h2_bits(__half2half2(x2));
          }
          tc::tmem_st16(ta + 16 * q4, a16);
        }
        tc::tmem_wait_st();
        tc::fence_before_sync();
        tc::mbar_arrive(&a_full[sa]);
      }
      it = nx;
      have = have_nx;
      rin = rnx;
    }
  } else if (warp < 8) {
    // ---------------- epilogue: thread = accumulator row = TMEM lane ----------------
    const int e = threadIdx.x - 128;
    const uint32_t lane_off = (uint32_t)(32 * (warp - 4)) << 16;
    int cur_tt = -1;
    Item it;
    bool qok = true;
    // one outcome for all four epilogue warps: they share named barriers below
    for (int i = 0; tc::bar_and(1, 128, next_item(p, iq, i, it, qok, false)); ++i) {
      const int ab = i % C::NACC, use = i / C::NACC;
      const int64_t tok0 = (int64_t)it.tt * NT;
      if (it.tt != cur_tt) {  // the token tile's scales (and targets)
        asm volatile("bar.sync 1, 128;\n" ::: "memory");
        if (e < NT) {
          if (MODE == 1) tgt_s[e] = tok0 + e < p.N ? __ldg(p.targets + tok0 + e) : -1;
          tsc_s[e] = tok0 + e < p.N ? __ldg(p.tsc + tok0 + e) : 1.f;
        }
        asm volatile("bar.sync 1, 128;\n" ::: "memory");
        cur_tt = it.tt;
      }
      const int64_t v = it.row0 + e;
      const bool live = v < it.row_end;
      const float sp = row_scale(load_row(p, v)).sp;  // loads overlap the wait below
      // one outcome for all four epilogue warps: they share named barriers below
      if (!tc::bar_and(1, 128, tc::mbar_wait(&acc_full[ab], use & 1, p.err))) break;
      tc::fence_after_sync();
      // The accumulator is read in batches of up to 32 columns into registers (all loads of
      // a batch in flight together); it is released as soon as the last batch is in
      // registers, before that batch is scaled and stored.
      constexpr int HC = NT < 32 ? NT : 32;
      // A part of a shared tile: the raw accumulator goes to this CTA's scratch slot, then
      // the tile's counter tells whether the other part is already there; the second part
      // finishes the tile from the two slots (their sum does not depend on the order).
      const float* mine = nullptr;
      const float* other = nullptr;
      if (it.part) {
        float* slot = p.scratch + (size_t)(blockIdx.x * 2 + (it.part == 1 ? 1 : 0)) * NT * 128 + e;
#pragma unroll 1
        for (int h = 0; h < NT / HC; ++h) {
          uint32_t r[HC / 16][16];
#pragma unroll
          for (int c = 0; c < HC / 16; ++c)
            tc::tmem_ld16_nowait(tbase + ab * NT + lane_off + h * HC + 16 * c, r[c]);
#pragma unroll
          for (int c = 0; c < HC / 16; ++c) tc::tmem_wait_ld(r[c]);
          if (h == NT / HC - 1) {
            tc::fence_before_sync();
            tc::mbar_arrive(&acc_empty[ab]);
          }
#pragma unroll
          for (int c = 0; c < HC / 16; ++c)
#pragma unroll
            for (int q = 0; q < 16; ++q) slot[(h * HC + 16 * c + q) * 128] = __uint_as_float(r[c][q]);
        }
        __threadfence();
        asm volatile("bar.sync 1, 128;\n" ::: "memory");
        if (e == 0) {
          grid_dependency_wait();  // the counters are zeroed by the prologue kernels
          *ep_flag = (int)atomicAdd(p.counters + it.vt, 1u);
        }
        asm volatile("bar.sync 1, 128;\n" ::: "memory");
        const bool second = *reinterpret_cast<volatile int*>(ep_flag) != 0;
        asm volatile("bar.sync 1, 128;\n" ::: "memory");  // the flag is reused
        if (!second) continue;
        __threadfence();
        mine = slot;
        other = p.scratch +
                (size_t)((blockIdx.x + (it.part == 1 ? 1 : -1)) * 2 + (it.part == 1 ? 0 : 1)) * NT * 128 + e;
      }
#pragma unroll 1
      for (int h = 0; h < NT / HC; ++h) {
        uint32_t r[HC / 16][16];
        if (mine) {
#pragma unroll
          for (int c = 0; c < HC / 16; ++c)
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int col = (h * HC + 16 * c + q) * 128;
              r[c][q] = __float_as_uint(__ldcg(mine + col) + __ldcg(other + col));
            }
        } else {
#pragma unroll
          for (int c = 0; c < HC / 16; ++c)
            tc::tmem_ld16_nowait(tbase + ab * NT + lane_off + h * HC + 16 * c, r[c]);
#pragma unroll
          for (int c = 0; c < HC / 16; ++c) tc::tmem_wait_ld(r[c]);
          if (h == NT / HC - 1) {
            tc::fence_before_sync();
            tc::mbar_arrive(&acc_empty[ab]);
          }
        }
#pragma unroll
        for (int c = 0; c < HC / 16; ++c) {
          const int c16 = h * (HC / 16) + c;  // 16-token chunk of the tile
          float y[16];
          const float4* ts4 = reinterpret_cast<const float4*>(tsc_s + 16 * c16);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {  // the logit of token q: accumulator x S'_v x 2^e_q
            const float4 f = ts4[q4];
            y[4 * q4 + 0] = __uint_as_float(r[c][4 * q4 + 0]) * sp * f.x;
            y[4 * q4 + 1] = __uint_as_float(r[c][4 * q4 + 1]) * sp * f.y;
            y[4 * q4 + 2] = __uint_as_float(r[c][4 * q4 + 2]) * sp * f.z;
            y[4 * q4 + 3] = __uint_as_float(r[c][4 * q4 + 3]) * sp * f.w;
          }
          if (MODE == 0) {
            if (live) {
              // token rows of the chunk below N, one pointer stepped by a row of Y
              const int64_t t16 = tok0 + 16 * c16;
              const int64_t nq = p.N - t16;
              float* yp = p.Y + t16 * p.V + v;
#pragma unroll
              for (int q = 0; q < 16; ++q) {
                if (q < nq) __stcs(yp, y[q]);  // streaming: Y does not displace the B image
                yp += p.V;
              }
            }
          } else {
            // ---- fused NLL: per token of the chunk, (max, sum exp) over the tile's rows ----
            const float NEG_INF = __int_as_float(0xff800000);
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              nll_y[q * 128 + e] = live ? y[q] : NEG_INF;
              const int tg = tgt_s[16 * c16 + q];
              if (live && tg == v) p.tlogit[tok0 + 16 * c16 + q] = y[q];
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
            const int64_t tok = tok0 + 16 * c16 + q;
            if (seg == 0 && tok < p.N) p.part[tok * p.n_vtiles + it.vt] = make_float2(m, sm);
            asm volatile("bar.sync 1, 128;\n" ::: "memory");
          }
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// The B image of the residual blocks: FP16 copy of H 2^-e_n (token scaling, see
// token_shift), for token tile tt of nt rows and 128-column block kb a contiguous nt x 128
// block at tc_image_offset (K-major, 128-byte swizzle).  Rows >= N are zero, and so are
// the nrb rank blocks after the nkb blocks of H, which the low-rank prologue then fills.
// One block per token row (grid-stride over rows): the row maximum first, then the
// conversion; tsc[n] = 2^e_n.  Non-finite entries set kErrRangeH.
__global__ void __launch_bounds__(256) convert_h_blocked_kernel(const uint16_t* __restrict__ H,
                                                                __half* __restrict__ Hb,
                                                                float* __restrict__ tsc,
                                                                int64_t N, int64_t Npad,
                                                                int64_t D, int64_t nkbt, int nt,
                                                                unsigned* counters, int64_t ncnt,
                                                                unsigned* err) {
  allow_dependent_launch();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < ncnt;
       i += (int64_t)gridDim.x * blockDim.x)
    counters[i] = 0u;
  __shared__ float red32[8];
  const int64_t chunks_per_row = nkbt * 16;  // 8 FP16 per chunk
  const int64_t hchunks = D / 8;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  bool bad = false;
  for (int64_t n = blockIdx.x; n < Npad; n += gridDim.x) {
    float m = 0.f;
    if (n < N)
      for (int64_t kc = threadIdx.x; kc < hchunks; kc += blockDim.x)
        m = fmaxf(m, bf16x8_absmax(__ldg(reinterpret_cast<const uint4*>(H + n * D + kc * 8))));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __syncthreads();  // red32 of the previous row has been read
    if (lane == 0) red32[warp] = m;
    __syncthreads();
    m = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red32[w]);
    const int e = token_shift(m);
    const float sc = ldexpf(1.f, -e);
    if (n < N && threadIdx.x == 0) tsc[n] = ldexpf(1.f, e);
    const int64_t tt = n / nt, nn = n - tt * nt;
    for (int64_t kc = threadIdx.x; kc < chunks_per_row; kc += blockDim.x) {
      uint4 out = make_uint4(0, 0, 0, 0);
      if (n < N && kc < hchunks) {
        const uint4 in = __ldg(reinterpret_cast<const uint4*>(H + n * D + kc * 8));
        const uint32_t w[4] = {in.x, in.y, in.z, in.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const __half2 h = __floats2half2_rn(__uint_as_float(w[k] << 16) * sc,
                                              __uint_as_float(w[k] & 0xFFFF0000u) * sc);
          o[k] = h2_bits(h);
          bad |= ((o[k] & 0x7C00u) == 0x7C00u) | ((o[k] & 0x7C000000u) == 0x7C000000u);
        }
        out = make_uint4(o[0], o[1], o[2], o[3]);
      }
      *reinterpret_cast<uint4*>(Hb + tc_image_offset(tt, kc >> 4, nkbt, nt, nn,
                                                     (int)(kc & 15) * 8)) = out;
    }
  }
  if (bad) atomicOr(err, kErrRangeH);
}

// Resident CTAs per SM of a kernel: registers (allocated per warp in units of 256), shared
// memory (plus the 1 KB the driver reserves per CTA), warps and tensor-memory columns.
int tc_residency(const cudaFuncAttributes& fa, size_t smem, int tmem_cols, int regs_sm,
                 int smem_sm) {
  const int warps = kTcThreads / 32;
  const int regs_warp = (fa.numRegs * 32 + 255) / 256 * 256;
  int occ = regs_sm / (regs_warp * warps);
  const int by_smem = smem_sm / (int)(smem + fa.sharedSizeBytes + 1024);
  if (by_smem < occ) occ = by_smem;
  if (64 / warps < occ) occ = 64 / warps;
  if (512 / tmem_cols < occ) occ = 512 / tmem_cols;
  return occ;
}

template <int NT, int CPC, int MODE>
cudaError_t launch_tc_cfg(const TcParams& p, cudaStream_t st) {
  const size_t smem = tc_smem_bytes<NT>(p.sb, p.spk, (int)(p.D >> p.g_shift), MODE == 1);
  auto kern = residual_tc_kernel<NT, CPC, MODE>;
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
  int occ = tc_residency(fa, smem, TcCfg<NT>::TMEM_COLS, regs_sm, smem_sm);
  if (occ < 1) occ = 1;
  int64_t items = p.n_vtiles * p.n_tok_tiles;
  int64_t grid = (int64_t)sms * occ;
  if (grid > items) grid = items;
  return launch_dependent(kern, grid, kTcThreads, smem, st, p);
}

template <int NT, int MODE>
cudaError_t launch_tc_nt(const TcParams& p, int g, cudaStream_t st) {
  if (g == 32) return launch_tc_cfg<NT, 4, MODE>(p, st);
  if (g == 64) return launch_tc_cfg<NT, 2, MODE>(p, st);
  return launch_tc_cfg<NT, 1, MODE>(p, st);
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

// First (B stages, packed stages) pair whose shared memory fits the budget; nt = 0 if none.
template <int NT>
TcPlan fit_rings(const int (*pairs)[2], int npairs, int G, bool nll, size_t budget) {
  for (int i = 0; i < npairs; ++i)
    if (tc_smem_bytes<NT>(pairs[i][0], pairs[i][1], G, nll) <= budget)
      return TcPlan{NT, pairs[i][0], 0, pairs[i][1]};
  return TcPlan{0, 0, 0, 0};
}

}  // namespace

TcPlan tc_plan(const Shapes& s, bool nll) {
  // Shared memory per SM is 228 KB with 1 KB reserved per CTA: two CTAs per SM take at
  // most 113 KB each.
  const size_t two_per_sm = 228 * 1024 / 2 - 1024;
  const int G = (int)(s.D / s.g);
  TcPlan pl = {0, 0, 0, 0};
  if (s.N > 64) {
    static const int p128[][2] = {{2, 4}, {2, 3}, {2, 2}};
    pl = fit_rings<128>(p128, 3, G, nll, two_per_sm);
  }
  if (!pl.nt) {
    static const int p16[][2] = {{8, 6}, {7, 6}, {6, 6}, {5, 6}, {4, 6}, {3, 6}, {2, 6}, {2, 4}};
    static const int p32[][2] = {{6, 6}, {5, 6}, {4, 6}, {3, 6}, {2, 6}, {2, 4}};
    static const int p64[][2] = {{4, 4}, {3, 4}, {2, 4}};
    if (s.N <= 16) pl = fit_rings<16>(p16, 8, G, nll, two_per_sm);
    else if (s.N <= 32) pl = fit_rings<32>(p32, 6, G, nll, two_per_sm);
    else pl = fit_rings<64>(p64, 3, G, nll, two_per_sm);
  }
  pl.nrb = (s.r_c + s.r_r + 31) / 32;
  return pl;
}

size_t tc_split_scratch_bytes(const Shapes& s, const TcPlan& plan) {
  if (plan.nt == 0 || s.N > plan.nt) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  // two CTAs per SM at most (tensor memory), two slots each
  return (size_t)2 * sms * 2 * plan.nt * 128 * 4;
}

cudaError_t launch_prologue_blocked(const uint16_t* H, const archead_head* head,
                                    const Shapes& s, const TcPlan& plan, __half* Hb, float* tsc,
                                    unsigned* counters, unsigned* err, cudaStream_t st,
                                    int* launches) {
  const int nt = plan.nt;
  const int64_t Npad = (s.N + nt - 1) / nt * nt;
  const int64_t nkbt = s.D / 128 + plan.nrb;
  int64_t blocks = Npad < 148 * 16 ? Npad : 148 * 16;  // one block per row (grid-stride)
  convert_h_blocked_kernel<<<(unsigned)(blocks < 1 ? 1 : blocks), 256, 0, st>>>(
      H, Hb, tsc, s.N, Npad, s.D, nkbt, nt, counters, counters ? (s.V + 127) / 128 : 0, err);
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_lowrank_t(H, head, s, nullptr, Hb, nt, nkbt, err, st, launches);
}

cudaError_t launch_residual_tc(const __half* Hb, const float* tsc, const archead_head* head,
                               const Shapes& s, const TcPlan& plan, float* Y,
                               const int32_t* targets,
                               float2* part, float* tlogit, float* scratch, unsigned* counters,
                               unsigned* err, cudaStream_t st, int* launches) {
  TcParams p;
  p.Hb = Hb;
  p.tsc = tsc;
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
  p.nrb = plan.nrb;
  p.rank_steps = (4 * (s.r_c + s.r_r) + 15) / 16;
  // factor rows as aligned words: both ranks multiples of 4 (bases are 16-byte aligned)
  p.a_words = (s.r_c % 4 == 0 && s.r_r % 4 == 0) ? 1 : 0;
  p.sb = plan.sb;
  p.spk = plan.sp;
  p.err = err;
  p.n_tok_tiles = (int)((s.N + plan.nt - 1) / plan.nt);
  {
    // a band's B image within about 48 MB, well inside the 126 MB L2
    const int64_t tile_bytes = (int64_t)plan.nt * (s.D + 128 * plan.nrb) * 2;
    int64_t band = (48ll << 20) / tile_bytes;
    if (band < 1) band = 1;
    if (band > p.n_tok_tiles) band = p.n_tok_tiles;
    p.tt_band = (int)band;
  }
  p.n_vtiles = (s.V + 127) / 128;
  p.split = (p.n_tok_tiles == 1 && scratch && counters) ? 1 : 0;
  p.dyn = (p.n_tok_tiles > 1 && counters && p.n_vtiles * p.n_tok_tiles < (1ll << 31)) ? 1 : 0;
  p.scratch = scratch;
  p.counters = counters;
  if (plan.nt == 0 || plan.sb < 2 || plan.sb > kMaxSB || plan.sp < 2 || plan.sp > kMaxSP)
    return cudaErrorInvalidValue;
  cudaError_t e = Y ? launch_tc_mode<0>(p, plan.nt, s.g, st)
                    : launch_tc_mode<1>(p, plan.nt, s.g, st);
  ++*launches;
  return e;
}

}  // namespace archead
