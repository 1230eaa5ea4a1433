// Switch auxiliary load-balancing loss and mean routing entropy from fp32
// router logits [T, E] (Switch notes sec. 2.2, "A Differentiable Load
// Balancing Loss", eqs. (4)-(6); the entropy is the routing entropy the
// TorchScale review tracks):
//   f_i = (1/T) #{x : argmax p(x) = i}      P_i = (1/T) sum_x p_i(x)
//   loss = alpha * E * sum_i f_i P_i        entropy = (1/T) sum_x H(p(x))
// with p(x) the softmax of eq. (1) over all E experts and the argmax taken on
// the fp32 logits, ties to the lower index (the top-1 choice).
//
// Pass 1 (reads the logits once): a warp per token, the logits of two tokens
// per warp loaded before either is reduced, E <= 256 logits held 8 per lane
// (coalesced); max/argmax and the softmax sum by shuffles; each lane
// accumulates p for its experts in fp32 over groups of 16 tokens and adds each
// group's sums to its double sums in shared memory (one conversion per 16
// tokens), the argmax is counted in shared memory, and H(p) = ln(s) -
// sum_e p_e (h_e - m) per token.  Each block (four per SM, one wave) writes its partial P[E], counts[E]
// and entropy sum, expert-major.  Pass 2: a block per expert adds that expert's partials
// (strided, then a fixed tree: deterministic); the last block to finish
// (a counter that pass 1 zeroes) forms sum_e f_e P_e and the entropy, in a
// fixed order.
#include <climits>
#include <cmath>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kAuxThreads = 256;  // 8 warps
constexpr int kAuxWarps = kAuxThreads / 32;
constexpr int kAuxInFlight = 2;  // tokens per warp whose logits are loaded together
constexpr int kAuxBlocksPerSm = 4;  // 4 x 256 threads x <= 64 registers fill the register file
constexpr int kAuxGroup = 16;       // tokens summed in fp32 before each double add

__global__ void __launch_bounds__(kAuxThreads, kAuxBlocksPerSm) aux_partial_kernel(
    int64_t T, int E, const float* __restrict__ logits, double* __restrict__ part_P,
    int32_t* __restrict__ part_cnt, double* __restrict__ part_H, unsigned* __restrict__ done) {
  __shared__ double s_P[kAuxWarps][256];
  __shared__ int s_cnt[256];
  __shared__ double s_H[kAuxWarps];
  dev::pdl_trigger();
  dev::pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < 256; e += kAuxThreads) s_cnt[e] = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) s_P[warp][lane + 32 * q] = 0.0;  // this lane's double sums
  if (blockIdx.x == 0 && threadIdx.x == 0) *done = 0u;  // pass 2's finishing counter
  __syncthreads();
  float grpP[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int in_grp = 0;
  double accH = 0.0;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kAuxWarps;
  // one token's logits, lane + 32 q for q < 8 (-inf past E)
  auto load = [&](int64_t t, float (&v)[8]) {
    const float* h = logits + t * E;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = lane + 32 * q;
      v[q] = e < E ? __ldg(h + e) : -INFINITY;
    }
  };
  // one token's softmax statistics
  auto token = [&](const float (&v)[8]) {
    // argmax with the lower index on ties: each lane scans its experts in
    // ascending order with a strict compare, then a shuffle reduction
    float bv = -INFINITY;
    int bi = INT_MAX;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = lane + 32 * q;
      if (e < E && v[q] > bv) { bv = v[q]; bi = e; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    const float m = bv;
    float ex[8];
    float s = 0.f, w = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const bool in = lane + 32 * q < E;
      ex[q] = in ? __expf(v[q] - m) : 0.f;
      s += ex[q];
      w += in ? ex[q] * (v[q] - m) : 0.f;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      s += __shfl_xor_sync(0xffffffffu, s, off);
      w += __shfl_xor_sync(0xffffffffu, w, off);
    }
    const float inv = 1.0f / s;
#pragma unroll
    for (int q = 0; q < 8; ++q) grpP[q] += ex[q] * inv;
    if (++in_grp == kAuxGroup) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        s_P[warp][lane + 32 * q] += static_cast<double>(grpP[q]);
        grpP[q] = 0.f;
      }
      in_grp = 0;
    }
    if (lane == 0) {
      if (bi < E) atomicAdd(&s_cnt[bi], 1);
      // H = -sum p ln p = ln s - sum p (h - m)
      accH += static_cast<double>(logf(s)) - static_cast<double>(w * inv);
    }
  };
  // the warp's tokens t, t + nwarps, ... in that order, kAuxInFlight at a time
  int64_t t = static_cast<int64_t>(blockIdx.x) * kAuxWarps + warp;
  for (; t + (kAuxInFlight - 1) * nwarps < T; t += kAuxInFlight * nwarps) {
    float v[kAuxInFlight][8];
#pragma unroll
    for (int u = 0; u < kAuxInFlight; ++u) load(t + u * nwarps, v[u]);
#pragma unroll
    for (int u = 0; u < kAuxInFlight; ++u) token(v[u]);
  }
  for (; t < T; t += nwarps) {
    float v[8];
    load(t, v);
    token(v);
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) s_P[warp][lane + 32 * q] += static_cast<double>(grpP[q]);
  if (lane == 0) s_H[warp] = accH;
  __syncthreads();
  // expert-major partials: pass 2's block for expert e reads its row coalesced
  for (int e = threadIdx.x; e < E; e += kAuxThreads) {
    double sum = 0.0;
    for (int wq = 0; wq < kAuxWarps; ++wq) sum += s_P[wq][e];
    part_P[static_cast<int64_t>(e) * gridDim.x + blockIdx.x] = sum;
    part_cnt[static_cast<int64_t>(e) * gridDim.x + blockIdx.x] = s_cnt[e];
  }
  if (threadIdx.x == 0) {
    double sum = 0.0;
    for (int wq = 0; wq < kAuxWarps; ++wq) sum += s_H[wq];
    part_H[blockIdx.x] = sum;
  }
}

// Pass 2: block e adds expert e's partials over the pass-1 blocks, stored
// expert-major (thread i
// takes blocks i, i + 256, ..., then a fixed tree), f_e = count / T,
// P_e = sum / T, fe_Pe[e] = f_e * P_e.  The block that finishes last (by the
// counter pass 1 zeroed) forms loss = alpha * E * sum_e f_e P_e and
// entropy = sum of the pass-1 entropy sums / T, both by fixed trees.
__global__ void __launch_bounds__(256, 1) aux_reduce_kernel(int64_t T, int E, int nblk, double alpha,
                                                         const double* __restrict__ part_P,
                                                         const int32_t* __restrict__ part_cnt,
                                                         const double* __restrict__ part_H,
                                                         double* fe_Pe, unsigned* done,
                                                         double* __restrict__ f_out,
                                                         double* __restrict__ P_out,
                                                         double* __restrict__ out) {
  __shared__ double s_p[256];
  __shared__ long long s_c[256];
  __shared__ double s_h[256];
  __shared__ bool s_last;
  dev::pdl_trigger();
  dev::pdl_wait();
  const int e = blockIdx.x;
  double p = 0.0;
  long long c = 0;
  const double* rowP = part_P + static_cast<int64_t>(e) * nblk;
  const int32_t* rowC = part_cnt + static_cast<int64_t>(e) * nblk;
  for (int b = threadIdx.x; b < nblk; b += 256) {
    p += rowP[b];
    c += rowC[b];
  }
  s_p[threadIdx.x] = p;
  s_c[threadIdx.x] = c;
  __syncthreads();
  for (int h = 128; h > 0; h >>= 1) {
    if (threadIdx.x < h) {
      s_p[threadIdx.x] += s_p[threadIdx.x + h];
      s_c[threadIdx.x] += s_c[threadIdx.x + h];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double Td = static_cast<double>(T);  // T = 0: every output is 0
    const double fe = T > 0 ? static_cast<double>(s_c[0]) / Td : 0.0;
    const double Pe = T > 0 ? s_p[0] / Td : 0.0;
    if (f_out) f_out[e] = fe;
    if (P_out) P_out[e] = Pe;
    fe_Pe[e] = fe * Pe;
    __threadfence();  // fe_Pe[e] visible before this block counts as done
    s_last = atomicAdd(done, 1u) == static_cast<unsigned>(E - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  double d = 0.0, hs = 0.0;
  for (int q = threadIdx.x; q < E; q += 256) d += __ldcg(fe_Pe + q);
  for (int b = threadIdx.x; b < nblk; b += 256) hs += part_H[b];
  s_p[threadIdx.x] = d;  // s_p[0] was read before the last barrier
  s_h[threadIdx.x] = hs;
  __syncthreads();
  for (int k = 128; k > 0; k >>= 1) {
    if (threadIdx.x < k) {
      s_p[threadIdx.x] += s_p[threadIdx.x + k];
      s_h[threadIdx.x] += s_h[threadIdx.x + k];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    out[0] = alpha * static_cast<double>(E) * s_p[0];
    out[1] = T > 0 ? s_h[0] / static_cast<double>(T) : 0.0;
  }
}

int aux_blocks(const moe_config& c) {
  const int64_t want = (c.T + kAuxWarps * 4 - 1) / (kAuxWarps * 4);  // >= 4 tokens per warp
  const int64_t cap = static_cast<int64_t>(num_sms()) * kAuxBlocksPerSm;  // one wave
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

}  // namespace

// per expert: P [nblk] double, then counts [nblk] int32 (expert-major); then the entropy sums [nblk]
// double; then f_e P_e [E] double; then pass 2's finishing counter
size_t aux_workspace_bytes(const moe_config& c) {
  const size_t nblk = static_cast<size_t>(aux_blocks(c));
  return align256(nblk * c.E * sizeof(double)) + align256(nblk * c.E * sizeof(int32_t)) +
         align256(nblk * sizeof(double)) + align256(static_cast<size_t>(c.E) * sizeof(double)) +
         align256(sizeof(unsigned));
}

int32_t launch_aux_loss(const moe_config& c, const float* logits, double alpha, double* out,
                        double* f, double* P, void* workspace, cudaStream_t s) {
  const int nblk = aux_blocks(c);
  const size_t bP = align256(static_cast<size_t>(nblk) * c.E * 8);
  const size_t bC = align256(static_cast<size_t>(nblk) * c.E * 4);
  const size_t bH = align256(static_cast<size_t>(nblk) * 8);
  char* ws = static_cast<char*>(workspace);
  double* part_P = reinterpret_cast<double*>(ws);
  int32_t* part_cnt = reinterpret_cast<int32_t*>(ws + bP);
  double* part_H = reinterpret_cast<double*>(ws + bP + bC);
  double* fe_Pe = reinterpret_cast<double*>(ws + bP + bC + bH);
  unsigned* done = reinterpret_cast<unsigned*>(ws + bP + bC + bH + align256(static_cast<size_t>(c.E) * 8));
  launch_pdl(aux_partial_kernel, dim3(static_cast<unsigned>(nblk)), dim3(kAuxThreads), 0, s, c.T,
             c.E, logits, part_P, part_cnt, part_H, done);
  int32_t rc = check_launch("aux_partial_kernel");
  if (rc != MOE_OK) return rc;
  launch_pdl(aux_reduce_kernel, dim3(static_cast<unsigned>(c.E)), dim3(256), 0, s, c.T, c.E, nblk,
             alpha, static_cast<const double*>(part_P), static_cast<const int32_t*>(part_cnt),
             static_cast<const double*>(part_H), fe_Pe, done, f, P, out);
  return check_launch("aux_reduce_kernel");
}

}  // namespace moe
