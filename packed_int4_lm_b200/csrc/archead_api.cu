// C ABI of the ARCHead packed LM-head library: argument validation, stream-ordered
// scratch, the per-device error word and kernel dispatch.  See include/archead.h.
#include <algorithm>
#include <mutex>

#include "archead_internal.cuh"

namespace archead {

// Device-side error word: one instance per device that loads the library.
static __device__ unsigned g_error_word;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  unsigned* err = nullptr;       // device address of g_error_word on this device
  cudaMemPool_t pool = nullptr;  // library-owned stream-ordered pool
  cudaStream_t copy = nullptr;   // device-to-host copies of archead_logits_host
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
thread_local int t_last_launches = 0;

// archead_profile: event pairs recorded around the residual kernel
constexpr int kProfCap = 16384;
struct Profile {
  bool on = false;
  int count = 0;
  cudaEvent_t* ev = nullptr;  // 2 * kProfCap, created lazily
} g_prof;

void prof_mark(int which, cudaStream_t st) {
  if (!g_prof.on || g_prof.count >= kProfCap) return;
  cudaEventRecord(g_prof.ev[2 * g_prof.count + which], st);
  if (which == 1) ++g_prof.count;
}

int current_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return ARCHEAD_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.ready) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_error_word) != cudaSuccess) return ARCHEAD_ERR_CUDA;
    if (cudaMemset(addr, 0, sizeof(unsigned)) != cudaSuccess) return ARCHEAD_ERR_CUDA;
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return ARCHEAD_ERR_CUDA;
    uint64_t keep = ~0ull;  // keep freed blocks cached in the pool between calls
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (cudaDeviceSynchronize() != cudaSuccess) return ARCHEAD_ERR_CUDA;
    s.err = static_cast<unsigned*>(addr);
    s.pool = pool;
    s.ready = true;
  }
  *out = &s;
  return ARCHEAD_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The non-blocking stream on which archead_logits_host copies Y to the host (created on
// first use, kept for the life of the process).
int copy_stream(DeviceState* ds, cudaStream_t* out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!ds->copy && cudaStreamCreateWithFlags(&ds->copy, cudaStreamNonBlocking) != cudaSuccess) {
    ds->copy = nullptr;
    cudaGetLastError();
    return ARCHEAD_ERR_CUDA;
  }
  *out = ds->copy;
  return ARCHEAD_OK;
}

// The rows [v0, v0 + rows) of a head as a head of its own (v0 a multiple of 128): every
// per-row array is row-major, and the device nibble layout is tile-major with 128 x D/2
// bytes per 128-row tile, so the view is the same pointers advanced by v0 rows.
archead_head head_rows(const archead_head& h, int64_t v0, int64_t rows) {
  archead_head s = h;
  s.V = rows;
  if (h.format == ARCHEAD_FMT_ROW8) {
    s.r_nib = h.r_nib + v0 * h.D;
    s.row_scale = h.row_scale + v0;
    return s;
  }
  s.r_nib = h.r_nib + v0 * (h.D / 2);
  s.r_code = h.r_code + v0 * (h.D / h.g);
  s.r_super = h.r_super + v0;
  if (h.Ac) s.Ac = h.Ac + v0 * h.r_c;
  if (h.sAc) s.sAc = h.sAc + v0;
  if (h.Aw) s.Aw = h.Aw + v0 * h.r_r;
  if (h.sAw) s.sAw = h.sAw + v0;
  return s;
}

// archead_logits_host splits the vocabulary into chunks of about this many bytes of Y (at
// most kMaxHostChunks, each a multiple of 128 rows) and copies each chunk's logits to the
// host while the next chunks are evaluated: the copy of 4 bytes per logit over the host
// link takes longer than the kernels for all but the smallest N.
constexpr size_t kHostChunkBytes = 3u << 20;
constexpr int kMaxHostChunks = 8;

int64_t host_chunk_rows(int64_t N, int64_t V) {
  const size_t yb = (size_t)N * V * 4;
  const int64_t c = (int64_t)std::min<size_t>(kMaxHostChunks, yb / kHostChunkBytes);
  if (c < 2 || V < 256) return V;
  return (int64_t)round_up((size_t)((V + c - 1) / c), 128);
}

int check_head(const archead_head* h, int64_t N, int64_t V, int64_t D, int r_c, int r_r,
               int g) {
  if (!h) return ARCHEAD_ERR_NULLPTR;
  if (h->V != V || h->D != D || h->r_c != r_c || h->r_r != r_r || h->g != g)
    return ARCHEAD_ERR_SHAPE;
  // V: the residual kernel's grid.y holds one 128-row vocabulary block each (<= 65535)
  if (N < 0 || N > 0x7fffffffLL || V < 1 || V > 65535LL * 128 || D < 128 || D % 128 != 0 ||
      D > (1LL << 20))
    return ARCHEAD_ERR_SHAPE;
  if (!(g == 32 || g == 64 || g == 128 || g == 256) || D % g != 0) return ARCHEAD_ERR_SHAPE;
  if (r_c < 0 || r_c > 128 || r_r < 0 || r_r > 128) return ARCHEAD_ERR_SHAPE;
  if (h->format == ARCHEAD_FMT_ROW8) {  // Row INT8: weights and row scales only
    if (r_c != 0 || r_r != 0) return ARCHEAD_ERR_SHAPE;
    if (!h->r_nib || !h->row_scale) return ARCHEAD_ERR_NULLPTR;
    if (!aligned(h->r_nib, 16) || !aligned(h->row_scale, 16)) return ARCHEAD_ERR_ALIGN;
    return ARCHEAD_OK;
  }
  if (h->format != ARCHEAD_FMT_SC4) return ARCHEAD_ERR_SHAPE;
  if (!h->r_nib || !h->r_code || !h->r_super) return ARCHEAD_ERR_NULLPTR;
  if (r_c > 0 && (!h->Ac || !h->sAc || !h->Bc || !h->sBc)) return ARCHEAD_ERR_NULLPTR;
  if (r_r > 0 && (!h->Aw || !h->sAw || !h->Bw || !h->sBw)) return ARCHEAD_ERR_NULLPTR;
  if (!aligned(h->r_nib, 16) || !aligned(h->r_code, 16) || !aligned(h->r_super, 16))
    return ARCHEAD_ERR_ALIGN;
  const void* f[] = {h->Ac, h->sAc, h->Bc, h->sBc, h->Aw, h->sAw, h->Bw, h->sBw};
  for (const void* p : f)
    if (p && !aligned(p, 16)) return ARCHEAD_ERR_ALIGN;
  return ARCHEAD_OK;
}

Shapes make_shapes(int64_t N, int64_t V, int64_t D, int r_c, int r_r, int g) {
  Shapes s;
  s.N = N;
  s.V = V;
  s.D = D;
  s.r_c = r_c;
  s.r_r = r_r;
  s.g = g;
  return s;
}

// Stream-ordered scratch: one allocation carved into aligned pieces.
struct Carve {
  size_t off = 0;
  size_t take(size_t bytes) {
    size_t o = off;
    off = round_up(off + (bytes ? bytes : 16), 256);
    return o;
  }
};

// A vocabulary shard of a larger head (archead_nll_partials): rows [v_begin, v_begin + V)
// of v_total; the NLL path then writes the per-token (max, sum exp, target logit) triples
// into partials instead of the NLL.
struct NllShard {
  int64_t v_begin, v_total;
  float* partials;
};

int run_dec(const uint16_t* H, const archead_head* head, float* Y, const int32_t* targets,
            float* nll, const Shapes& s, const DecPlan& pl, DeviceState* ds, cudaStream_t st,
            const NllShard* shard) {
  int launches = 0;
  const int RR = s.r_c + s.r_r;
  const bool nll_mode = nll != nullptr || shard != nullptr;
  const int64_t nvt = (s.V + 127) / 128;
  Carve cv;
  const size_t o_img = cv.take(dec_image_bytes(s, pl));
  const size_t o_t = cv.take((size_t)s.N * RR * 4);
  const size_t o_cnt = cv.take((size_t)nvt * 4);
  const size_t o_scr = cv.take(dec_partial_bytes(pl));
  const size_t o_part = nll_mode ? cv.take((size_t)s.N * nvt * 8) : 0;
  const size_t o_tl = nll_mode ? cv.take((size_t)s.N * 4) : 0;
  const size_t o_tloc = shard ? cv.take((size_t)s.N * 4) : 0;
  void* base = nullptr;
  if (cudaMallocFromPoolAsync(&base, cv.off, ds->pool, st) != cudaSuccess) {
    cudaGetLastError();
    return ARCHEAD_ERR_NOMEM;
  }
  char* b = static_cast<char*>(base);
  __half* img = reinterpret_cast<__half*>(b + o_img);
  float* t = reinterpret_cast<float*>(b + o_t);
  unsigned* cnt = reinterpret_cast<unsigned*>(b + o_cnt);
  float4* scr = reinterpret_cast<float4*>(b + o_scr);
  float2* part = nll_mode ? reinterpret_cast<float2*>(b + o_part) : nullptr;
  float* tl = nll_mode ? reinterpret_cast<float*>(b + o_tl) : nullptr;
  int32_t* tloc = shard ? reinterpret_cast<int32_t*>(b + o_tloc) : nullptr;
  cudaError_t e = cudaSuccess;
  if (shard)  // shard-local targets and zeroed target logits, before the prologue
    e = launch_nll_shard_prep(targets, s.N, shard->v_begin, s.V, shard->v_total, tloc, tl,
                              ds->err, st, &launches);
  const int32_t* tg = shard ? tloc : targets;
  if (e == cudaSuccess)
    e = launch_dec_prologue(H, head, s, pl, img, t, cnt, ds->err, st, &launches);
  if (e == cudaSuccess) {
    prof_mark(0, st);
    e = launch_residual_dec(img, t, head, s, pl, nll_mode ? nullptr : Y, tg, part, tl, scr,
                            cnt, ds->err, st, &launches);
    prof_mark(1, st);
    if (e == cudaSuccess && nll_mode)
      e = shard ? launch_nll_partials(part, tl, s, shard->partials, st, &launches)
                : launch_nll_combine(part, tl, targets, s, nll, ds->err, st, &launches);
  }
  cudaFreeAsync(base, st);
  if (e != cudaSuccess) return ARCHEAD_ERR_CUDA;
  t_last_launches = launches;
  return ARCHEAD_OK;
}

int run(const uint16_t* H, const archead_head* head, float* Y, const int32_t* targets,
        float* nll, const Shapes& s, cudaStream_t st, const NllShard* shard = nullptr) {
  DeviceState* ds;
  int rc = current_state(&ds);
  if (rc) return rc;
  int launches = 0;
  const int RR = s.r_c + s.r_r;
  const bool nll_mode = nll != nullptr || shard != nullptr;
  // N <= 16: the persistent decode kernel with H resident in shared memory, when its plan
  // fits; larger N: the tensor-memory (tcgen05) kernel when its shared-memory rings fit;
  // other shapes: the token-block warp-MMA kernel.  All three have a fused
  // split-vocabulary NLL epilogue.
  // Row INT8 heads run on the token-block warp-MMA kernel only
  const bool row8 = head->format == ARCHEAD_FMT_ROW8;
  const DecPlan dplan = row8 ? DecPlan{0, 0, 0} : dec_plan(s, nll_mode);
  if (dplan.nt8 > 0) return run_dec(H, head, Y, targets, nll, s, dplan, ds, st, shard);
  const TcPlan plan = s.N > 8 && !row8 ? tc_plan(s, nll_mode) : TcPlan{0, 0, 0, 0};
  const bool use_tc = plan.nt > 0;
  const int64_t tb = use_tc ? plan.nt : residual_token_block(s.N);
  const int64_t Npad = (s.N + tb - 1) / tb * tb;
  const int nvblk = residual_gemm_vblocks(s);
  Carve cv;
  // tcgen05: the B image holds H and the rank blocks; warp MMAs: FP16 H plus FP32 t
  const size_t o_hh = cv.take((size_t)Npad * (s.D + (use_tc ? 128 * plan.nrb : 0)) * 2);
  const size_t o_t = cv.take(use_tc ? 0 : (size_t)s.N * RR * 4);
  const size_t o_tsc = cv.take((size_t)s.N * 4);  // token scales 2^e_n
  const size_t o_part = nll_mode ? cv.take((size_t)s.N * nvblk * 8) : 0;
  const size_t o_tl = nll_mode ? cv.take((size_t)s.N * 4) : 0;
  // a single token tile is split evenly over the CTAs (partials + per-tile counters)
  const size_t split_bytes = use_tc ? tc_split_scratch_bytes(s, plan) : 0;
  const size_t o_scr = split_bytes ? cv.take(split_bytes) : 0;
  // per-tile counters of a split launch, or the work counter of the dynamic item order
  const size_t o_cnt = use_tc ? cv.take((size_t)((s.V + 127) / 128) * 4) : 0;
  const size_t o_tloc = shard ? cv.take((size_t)s.N * 4) : 0;
  void* base = nullptr;
  if (cudaMallocFromPoolAsync(&base, cv.off, ds->pool, st) != cudaSuccess) {
    cudaGetLastError();
    return ARCHEAD_ERR_NOMEM;
  }
  char* b = static_cast<char*>(base);
  __half* Hh = reinterpret_cast<__half*>(b + o_hh);
  float* scr = split_bytes ? reinterpret_cast<float*>(b + o_scr) : nullptr;
  unsigned* cnt = use_tc ? reinterpret_cast<unsigned*>(b + o_cnt) : nullptr;
  float* t = reinterpret_cast<float*>(b + o_t);
  float* tsc = reinterpret_cast<float*>(b + o_tsc);
  int32_t* tloc = shard ? reinterpret_cast<int32_t*>(b + o_tloc) : nullptr;
  cudaError_t e = cudaSuccess;
  if (shard)  // shard-local targets and zeroed target logits, before the prologue
    e = launch_nll_shard_prep(targets, s.N, shard->v_begin, s.V, shard->v_total, tloc,
                              reinterpret_cast<float*>(b + o_tl), ds->err, st, &launches);
  const int32_t* tg = shard ? tloc : targets;
  if (e == cudaSuccess)
    e = use_tc ? launch_prologue_blocked(H, head, s, plan, Hh, tsc, cnt, ds->err, st, &launches)
               : launch_prologue(H, head, s, Npad, Hh, t, tsc, ds->err, st, &launches);
  if (e == cudaSuccess) {
    if (use_tc) {
      float2* part = nll_mode ? reinterpret_cast<float2*>(b + o_part) : nullptr;
      float* tl = nll_mode ? reinterpret_cast<float*>(b + o_tl) : nullptr;
      prof_mark(0, st);
      e = launch_residual_tc(Hh, tsc, head, s, plan, nll_mode ? nullptr : Y, tg, part, tl, scr, cnt,
                             ds->err, st, &launches);
      prof_mark(1, st);
      if (e == cudaSuccess && nll_mode)
        e = shard ? launch_nll_partials(part, tl, s, shard->partials, st, &launches)
                  : launch_nll_combine(part, tl, targets, s, nll, ds->err, st, &launches);
    } else if (!nll_mode) {
      prof_mark(0, st);
      e = launch_residual_gemm(Hh, t, tsc, head, s, Y, nullptr, nullptr, nullptr, st, &launches, 0);
      prof_mark(1, st);
    } else {
      float2* part = reinterpret_cast<float2*>(b + o_part);
      float* tl = reinterpret_cast<float*>(b + o_tl);
      prof_mark(0, st);
      e = launch_residual_gemm(Hh, t, tsc, head, s, nullptr, tg, part, tl, st, &launches, 1);
      prof_mark(1, st);
      if (e == cudaSuccess)
        e = shard ? launch_nll_partials(part, tl, s, shard->partials, st, &launches)
                  : launch_nll_combine(part, tl, targets, s, nll, ds->err, st, &launches);
    }
  }
  cudaFreeAsync(base, st);
  if (e != cudaSuccess) return ARCHEAD_ERR_CUDA;
  t_last_launches = launches;
  return ARCHEAD_OK;
}

}  // namespace

// Argument validation shared with other entry points (same checks as archead_logits).
int validate_head_args(const archead_head* head, int64_t N, int64_t V, int64_t D, int r_c,
                       int r_r, int g) {
  return check_head(head, N, V, D, r_c, r_r, g);
}

// Device address of this device's error word (the device must be current).
unsigned* error_word_address() {
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_error_word) != cudaSuccess) return nullptr;
  return static_cast<unsigned*>(addr);
}

}  // namespace archead

using namespace archead;

extern "C" {

int archead_abi_version(void) { return ARCHEAD_ABI_VERSION; }

int archead_last_launches(void) { return t_last_launches; }

const char* archead_strerror(int status) {
  switch (status) {
    case ARCHEAD_OK: return "ok";
    case ARCHEAD_ERR_NULLPTR: return "a required pointer is NULL";
    case ARCHEAD_ERR_ALIGN: return "a pointer is not suitably aligned (16 bytes)";
    case ARCHEAD_ERR_SHAPE: return "sizes disagree with the head or break a limit";
    case ARCHEAD_ERR_RANGE_H:
      return "an entry of H is not finite, or a scaled rank product exceeds the FP16 range";
    case ARCHEAD_ERR_TARGET: return "a target id is outside [0, V)";
    case ARCHEAD_ERR_TIMEOUT: return "a bounded device wait gave up";
    case ARCHEAD_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    case ARCHEAD_ERR_UNSUPPORTED: return "unsupported device or configuration";
    case ARCHEAD_ERR_NOMEM: return "stream-ordered device allocation failed";
    default: return "unknown status";
  }
}

int archead_logits(const uint16_t* H, const archead_head* head, float* Y, int64_t N,
                   int64_t V, int64_t D, int r_c, int r_r, int g, void* stream) {
  int rc = check_head(head, N, V, D, r_c, r_r, g);
  if (rc) return rc;
  if (N == 0) {
    t_last_launches = 0;
    return ARCHEAD_OK;
  }
  if (!H || !Y) return ARCHEAD_ERR_NULLPTR;
  if (!aligned(H, 16) || !aligned(Y, 4)) return ARCHEAD_ERR_ALIGN;
  return run(H, head, Y, nullptr, nullptr, make_shapes(N, V, D, r_c, r_r, g),
             static_cast<cudaStream_t>(stream));
}

int archead_nll(const uint16_t* H, const archead_head* head, const int32_t* targets,
                float* nll_out, int64_t N, int64_t V, int64_t D, int r_c, int r_r, int g,
                void* stream) {
  int rc = check_head(head, N, V, D, r_c, r_r, g);
  if (rc) return rc;
  if (N == 0) {
    t_last_launches = 0;
    return ARCHEAD_OK;
  }
  if (!H || !targets || !nll_out) return ARCHEAD_ERR_NULLPTR;
  if (!aligned(H, 16) || !aligned(targets, 4) || !aligned(nll_out, 4)) return ARCHEAD_ERR_ALIGN;
  return run(H, head, nullptr, targets, nll_out, make_shapes(N, V, D, r_c, r_r, g),
             static_cast<cudaStream_t>(stream));
}

int archead_nll_partials(const uint16_t* H, const archead_head* head, const int32_t* targets,
                         int64_t v_begin, int64_t v_total, float* partials, int64_t N,
                         int64_t V, int64_t D, int r_c, int r_r, int g, void* stream) {
  int rc = check_head(head, N, V, D, r_c, r_r, g);
  if (rc) return rc;
  if (v_begin < 0 || v_total < V || v_begin > v_total - V || v_total > 0x7fffffffLL)
    return ARCHEAD_ERR_SHAPE;
  if (N == 0) {
    t_last_launches = 0;
    return ARCHEAD_OK;
  }
  if (!H || !targets || !partials) return ARCHEAD_ERR_NULLPTR;
  if (!aligned(H, 16) || !aligned(targets, 4) || !aligned(partials, 4)) return ARCHEAD_ERR_ALIGN;
  const NllShard shard = {v_begin, v_total, partials};
  return run(H, head, nullptr, targets, nullptr, make_shapes(N, V, D, r_c, r_r, g),
             static_cast<cudaStream_t>(stream), &shard);
}

int archead_nll_merge(const float* partials, int G, int64_t N, float* nll_out, void* stream) {
  if (N < 0 || N > 0x7fffffffLL || G < 1 || G > 65536) return ARCHEAD_ERR_SHAPE;
  if (N == 0) {
    t_last_launches = 0;
    return ARCHEAD_OK;
  }
  if (!partials || !nll_out) return ARCHEAD_ERR_NULLPTR;
  if (!aligned(partials, 4) || !aligned(nll_out, 4)) return ARCHEAD_ERR_ALIGN;
  if (launch_nll_merge(partials, G, N, nll_out, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return ARCHEAD_ERR_CUDA;
  t_last_launches = 1;
  return ARCHEAD_OK;
}

int archead_agreement(const uint16_t* H, const archead_head* head, const float* Y_dense,
                      int k, int32_t* topk_out, int32_t* top1_dense_out, float* kl_out,
                      float* lse_out, int64_t N, int64_t V, int64_t D, int r_c, int r_r, int g,
                      void* stream) {
  int rc = check_head(head, N, V, D, r_c, r_r, g);
  if (rc) return rc;
  if (k < 1 || k > 16) return ARCHEAD_ERR_SHAPE;
  if (N == 0) {
    t_last_launches = 0;
    return ARCHEAD_OK;
  }
  if (!H || !Y_dense || !topk_out || !top1_dense_out || !kl_out) return ARCHEAD_ERR_NULLPTR;
  if (!aligned(H, 16) || !aligned(Y_dense, 4) || !aligned(topk_out, 4) ||
      !aligned(top1_dense_out, 4) || !aligned(kl_out, 4) || (lse_out && !aligned(lse_out, 4)))
    return ARCHEAD_ERR_ALIGN;
  DeviceState* ds;
  rc = current_state(&ds);
  if (rc) return rc;
  const Shapes s = make_shapes(N, V, D, r_c, r_r, g);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t tb = residual_token_block(N);
  const int64_t Npad = (N + tb - 1) / tb * tb;
  const int64_t nvblk = residual_gemm_vblocks(s);
  Carve cv;
  const size_t o_hh = cv.take((size_t)Npad * D * 2);
  const size_t o_t = cv.take((size_t)N * (r_c + r_r) * 4);
  const size_t o_tsc = cv.take((size_t)N * 4);
  const size_t o_st = cv.take((size_t)N * nvblk * 6 * 4);
  const size_t o_kv = cv.take((size_t)N * nvblk * k * 4);
  const size_t o_ki = cv.take((size_t)N * nvblk * k * 4);
  void* base = nullptr;
  if (cudaMallocFromPoolAsync(&base, cv.off, ds->pool, st) != cudaSuccess) {
    cudaGetLastError();
    return ARCHEAD_ERR_NOMEM;
  }
  char* b = static_cast<char*>(base);
  int launches = 0;
  __half* Hh = reinterpret_cast<__half*>(b + o_hh);
  float* t = reinterpret_cast<float*>(b + o_t);
  float* tsc = reinterpret_cast<float*>(b + o_tsc);
  cudaError_t e = launch_prologue(H, head, s, Npad, Hh, t, tsc, ds->err, st, &launches);
  if (e == cudaSuccess)
    e = launch_agreement(Hh, t, tsc, head, s, Y_dense, k, reinterpret_cast<float*>(b + o_st),
                         reinterpret_cast<float*>(b + o_kv), reinterpret_cast<int*>(b + o_ki),
                         topk_out, top1_dense_out, kl_out, lse_out, st, &launches);
  cudaFreeAsync(base, st);
  if (e != cudaSuccess) return ARCHEAD_ERR_CUDA;
  t_last_launches = launches;
  return ARCHEAD_OK;
}

int archead_logits_host(const uint16_t* H_host, const archead_head* head, float* Y_host,
                        int64_t N, int64_t V, int64_t D, int r_c, int r_r, int g,
                        void* stream) {
  int rc = check_head(head, N, V, D, r_c, r_r, g);
  if (rc) return rc;
  if (N == 0) return ARCHEAD_OK;
  if (!H_host || !Y_host) return ARCHEAD_ERR_NULLPTR;
  DeviceState* ds;
  rc = current_state(&ds);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t hb = (size_t)N * D * 2, yb = (size_t)N * V * 4;
  void* base = nullptr;
  const size_t yoff = round_up(hb, 256);
  if (cudaMallocFromPoolAsync(&base, yoff + yb, ds->pool, st) != cudaSuccess) {
    cudaGetLastError();
    return ARCHEAD_ERR_NOMEM;
  }
  uint16_t* Hd = static_cast<uint16_t*>(base);
  float* Yd = reinterpret_cast<float*>(static_cast<char*>(base) + yoff);
  rc = ARCHEAD_OK;
  if (cudaMemcpyAsync(Hd, H_host, hb, cudaMemcpyHostToDevice, st) != cudaSuccess)
    rc = ARCHEAD_ERR_CUDA;
  const int64_t rows = host_chunk_rows(N, V);
  if (rows >= V) {
    if (!rc) rc = archead_logits(Hd, head, Yd, N, V, D, r_c, r_r, g, stream);
    if (!rc && cudaMemcpyAsync(Y_host, Yd, yb, cudaMemcpyDeviceToHost, st) != cudaSuccess)
      rc = ARCHEAD_ERR_CUDA;
  } else {
    // chunk i: its kernels on `stream` write the N x vc block Yd + N v0 (its own row-major
    // logits), an event marks their end, and the copy stream waits for it and copies the
    // block into columns [v0, v0 + vc) of Y_host
    cudaStream_t cs = nullptr;
    cudaEvent_t ev[kMaxHostChunks + 1];
    int nev = 0;
    if (!rc) rc = copy_stream(ds, &cs);
    while (!rc && nev <= kMaxHostChunks) {
      if (cudaEventCreateWithFlags(&ev[nev], cudaEventDisableTiming) != cudaSuccess)
        rc = ARCHEAD_ERR_CUDA;
      else
        ++nev;
    }
    int launches = 0, i = 0;
    for (int64_t v0 = 0; !rc && v0 < V; v0 += rows, ++i) {
      const int64_t vc = std::min(rows, V - v0);
      const archead_head part = head_rows(*head, v0, vc);
      float* Yc = Yd + N * v0;
      rc = archead_logits(Hd, &part, Yc, N, vc, D, r_c, r_r, g, stream);
      if (rc) break;
      launches += t_last_launches;
      if (cudaEventRecord(ev[i], st) != cudaSuccess ||
          cudaStreamWaitEvent(cs, ev[i], 0) != cudaSuccess ||
          cudaMemcpy2DAsync(Y_host + v0, (size_t)V * 4, Yc, (size_t)vc * 4, (size_t)vc * 4,
                            (size_t)N, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
        rc = ARCHEAD_ERR_CUDA;
    }
    // the staging buffer goes back to the pool on `stream` only after the last copy
    if (cs && nev == kMaxHostChunks + 1 &&
        (cudaEventRecord(ev[kMaxHostChunks], cs) != cudaSuccess ||
         cudaStreamWaitEvent(st, ev[kMaxHostChunks], 0) != cudaSuccess)) {
      cudaStreamSynchronize(cs);
      if (!rc) rc = ARCHEAD_ERR_CUDA;
    }
    if (cs && nev < kMaxHostChunks + 1) cudaStreamSynchronize(cs);
    if (!rc) t_last_launches = launches;
    for (int j = 0; j < nev; ++j) cudaEventDestroy(ev[j]);
  }
  cudaFreeAsync(base, st);
  if (cudaStreamSynchronize(st) != cudaSuccess && !rc) rc = ARCHEAD_ERR_CUDA;
  return rc;
}

int archead_nll_host(const uint16_t* H_host, const archead_head* head,
                     const int32_t* targets_host, float* nll_host, int64_t N, int64_t V,
                     int64_t D, int r_c, int r_r, int g, void* stream) {
  int rc = check_head(head, N, V, D, r_c, r_r, g);
  if (rc) return rc;
  if (N == 0) return ARCHEAD_OK;
  if (!H_host || !targets_host || !nll_host) return ARCHEAD_ERR_NULLPTR;
  DeviceState* ds;
  rc = current_state(&ds);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t hb = (size_t)N * D * 2, tb = (size_t)N * 4;
  const size_t toff = round_up(hb, 256), noff = toff + round_up(tb, 256);
  void* base = nullptr;
  if (cudaMallocFromPoolAsync(&base, noff + tb, ds->pool, st) != cudaSuccess) {
    cudaGetLastError();
    return ARCHEAD_ERR_NOMEM;
  }
  char* b = static_cast<char*>(base);
  uint16_t* Hd = reinterpret_cast<uint16_t*>(b);
  int32_t* Td = reinterpret_cast<int32_t*>(b + toff);
  float* Nd = reinterpret_cast<float*>(b + noff);
  rc = ARCHEAD_OK;
  if (cudaMemcpyAsync(Hd, H_host, hb, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(Td, targets_host, tb, cudaMemcpyHostToDevice, st) != cudaSuccess)
    rc = ARCHEAD_ERR_CUDA;
  if (!rc) rc = archead_nll(Hd, head, Td, Nd, N, V, D, r_c, r_r, g, stream);
  if (!rc && cudaMemcpyAsync(nll_host, Nd, tb, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    rc = ARCHEAD_ERR_CUDA;
  cudaFreeAsync(base, st);
  if (cudaStreamSynchronize(st) != cudaSuccess && !rc) rc = ARCHEAD_ERR_CUDA;
  return rc;
}

int archead_repack_residual(const uint8_t* canon, uint8_t* dev, int64_t V, int64_t D,
                            void* stream) {
  if (!canon || !dev) return ARCHEAD_ERR_NULLPTR;
  if (V < 1 || V > 0x7fffffffLL || D < 128 || D % 128 != 0) return ARCHEAD_ERR_SHAPE;
  if (!aligned(canon, 16) || !aligned(dev, 16)) return ARCHEAD_ERR_ALIGN;
  const char* c0 = reinterpret_cast<const char*>(canon);
  const char* d0 = reinterpret_cast<const char*>(dev);
  const size_t nc = (size_t)V * D / 2, nd = (size_t)((V + 127) / 128 * 128) * D / 2;
  if (c0 < d0 + nd && d0 < c0 + nc) return ARCHEAD_ERR_SHAPE;  // overlapping buffers
  return launch_repack(canon, dev, V, D, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? ARCHEAD_OK
             : ARCHEAD_ERR_CUDA;
}

int archead_dequant(const archead_head* head, int64_t row0, int64_t nrows, float* R_out,
                    float* Ac_out, float* Aw_out, float* Bc_out, float* Bw_out,
                    void* stream) {
  if (!head) return ARCHEAD_ERR_NULLPTR;
  int rc = check_head(head, 0, head->V, head->D, head->r_c, head->r_r, head->g);
  if (rc) return rc;
  if (head->format != ARCHEAD_FMT_SC4) return ARCHEAD_ERR_UNSUPPORTED;
  if (row0 < 0 || nrows < 0 || row0 + nrows > head->V) return ARCHEAD_ERR_SHAPE;
  return launch_dequant(head, row0, nrows, R_out, Ac_out, Aw_out, Bc_out, Bw_out,
                        static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? ARCHEAD_OK
             : ARCHEAD_ERR_CUDA;
}

int archead_profile(int enable) {
  if (enable) {
    if (!g_prof.ev) {
      g_prof.ev = new cudaEvent_t[2 * kProfCap];
      for (int i = 0; i < 2 * kProfCap; ++i)
        if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) return ARCHEAD_ERR_CUDA;
    }
    g_prof.count = 0;
  }
  g_prof.on = enable != 0;
  return ARCHEAD_OK;
}

int archead_profile_read(double* total_ms, int* count) {
  double tot = 0.0;
  for (int i = 0; i < g_prof.count; ++i) {
    float ms = 0.f;
    if (cudaEventSynchronize(g_prof.ev[2 * i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) != cudaSuccess)
      return ARCHEAD_ERR_CUDA;
    tot += ms;
  }
  if (total_ms) *total_ms = tot;
  if (count) *count = g_prof.count;
  return ARCHEAD_OK;
}

int archead_test_hooks(long long wait_limit_cycles, int stall_cta) {
#ifdef ARCHEAD_TEST_HOOKS
  if (wait_limit_cycles < 1) return ARCHEAD_ERR_SHAPE;
  set_dec_test_hooks(wait_limit_cycles, stall_cta);
  return ARCHEAD_OK;
#else
  (void)wait_limit_cycles;
  (void)stall_cta;
  return ARCHEAD_ERR_UNSUPPORTED;
#endif
}

int archead_check(void* stream) {
  DeviceState* ds;
  int rc = current_state(&ds);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return ARCHEAD_ERR_CUDA;
  unsigned w = 0;
  if (cudaMemcpy(&w, ds->err, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess)
    return ARCHEAD_ERR_CUDA;
  if (w && cudaMemset(ds->err, 0, sizeof(unsigned)) != cudaSuccess) return ARCHEAD_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return ARCHEAD_ERR_CUDA;
  if (w & kErrRangeH) return ARCHEAD_ERR_RANGE_H;
  if (w & kErrTarget) return ARCHEAD_ERR_TARGET;
  if (w & kErrTimeout) return ARCHEAD_ERR_TIMEOUT;
  return ARCHEAD_OK;
}

}  // extern "C"
