// Vocabulary-parallel NLL (ARCHead Sec. 5, per-token cross-entropy in nats).
//
// With the head's V-indexed components split into row shards (one per GPU), every token's
//   nll = logsumexp_v Y[n, v] - Y[n, target]
// decomposes over shards k as  M = max_k m_k,  S = sum_k s_k exp(m_k - M),  nll = M +
// log S - y_t, where (m_k, s_k) are the shard's split-vocabulary log-sum-exp partials and
// y_t the target's logit from the one shard that owns the target row.  The main kernels'
// fused NLL mode already produces per-tile (max, sum exp) partials and the target logit;
// here a shard reduces them to one (m, s, y) triple per token (the target logit is 0 in
// shards that do not own it), and the merge combines G triples in shard order.  Between
// the two steps the triples cross GPUs once (an all-gather of 3 N floats per GPU).
#include "archead_internal.cuh"

namespace archead {
namespace {

// Shard-local targets: t - v_begin for targets in [v_begin, v_begin + V), else -1 (which
// matches no row); the shard's target logits start at 0.  Targets outside [0, v_total)
// set kErrTarget.
__global__ void __launch_bounds__(256) nll_shard_prep_kernel(
    const int32_t* __restrict__ targets, int64_t N, int64_t v_begin, int64_t V,
    int64_t v_total, int32_t* __restrict__ tloc, float* __restrict__ tlogit, unsigned* err) {
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < N;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = targets[i];
    const bool invalid = t < 0 || t >= v_total;
    bad |= invalid;
    tloc[i] = (!invalid && t >= v_begin && t < v_begin + V) ? (int32_t)(t - v_begin) : -1;
    tlogit[i] = 0.f;
  }
  if (bad) atomicOr(err, kErrTarget);
}

// One warp per token: the shard's (max, sum exp) over its per-tile partials, and the
// target logit.
__global__ void __launch_bounds__(256) nll_partials_kernel(const float2* __restrict__ part,
                                                           const float* __restrict__ tlogit,
                                                           int64_t N, int nvblk,
                                                           float* __restrict__ out) {
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
    out[3 * n] = m;
    out[3 * n + 1] = s;
    out[3 * n + 2] = tlogit[n];
  }
}

// One thread per token: G shard triples [G][N][3], combined in shard order.
__global__ void __launch_bounds__(256) nll_merge_kernel(const float* __restrict__ partials,
                                                        int G, int64_t N,
                                                        float* __restrict__ nll) {
  const int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (n >= N) return;
  const float NEG_INF = __int_as_float(0xff800000);
  float M = NEG_INF;
  for (int k = 0; k < G; ++k) M = fmaxf(M, partials[(k * N + n) * 3]);
  float S = 0.f, yt = 0.f;
  for (int k = 0; k < G; ++k) {
    const float* q = partials + (k * N + n) * 3;
    if (q[0] != NEG_INF) S += q[1] * expf(q[0] - M);
    yt += q[2];
  }
  nll[n] = M + logf(S) - yt;
}

}  // namespace

cudaError_t launch_nll_shard_prep(const int32_t* targets, int64_t N, int64_t v_begin,
                                  int64_t V, int64_t v_total, int32_t* tloc, float* tlogit,
                                  unsigned* err, cudaStream_t st, int* launches) {
  int64_t blocks = (N + 255) / 256;
  if (blocks > 148 * 4) blocks = 148 * 4;
  nll_shard_prep_kernel<<<(unsigned)(blocks < 1 ? 1 : blocks), 256, 0, st>>>(
      targets, N, v_begin, V, v_total, tloc, tlogit, err);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_nll_partials(const float2* part, const float* tlogit, const Shapes& s,
                                float* out, cudaStream_t st, int* launches) {
  const int nvblk = residual_gemm_vblocks(s);
  nll_partials_kernel<<<(unsigned)((s.N + 7) / 8), 256, 0, st>>>(part, tlogit, s.N, nvblk,
                                                                 out);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_nll_merge(const float* partials, int G, int64_t N, float* nll,
                             cudaStream_t st) {
  nll_merge_kernel<<<(unsigned)((N + 255) / 256), 256, 0, st>>>(partials, G, N, nll);
  return cudaGetLastError();
}

}  // namespace archead
