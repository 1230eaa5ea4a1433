// Routing: fp32 router (SIMT), softmax gate + top-k, Random Routed Experts,
// and the capacity-bounded slot assignment.
//
// Gate and top-k (Switch notes sec. 2.1, eq. 1): one warp per token holds the
// token's E <= 256 logits (8 per lane, coalesced), finds the largest with a
// shuffle reduction ordered by (value desc, index asc), the second largest
// the same way with the first excluded, and the softmax denominator
// sum_j exp(h_j - max) with a shuffle sum; gate = exp(h_i - max) / sum.
//
// Slot assignment (sec. 2.2, eq. 3 and the drop rule), in token order:
//   rank kernel     each 1024-assignment block ranks its choices per expert:
//                   __match_any_sync groups the lanes that chose the same
//                   expert, __popc of the lower peers gives the rank inside
//                   the warp, and per-warp counts are prefix-summed in shared
//                   memory across the 32 warps; block totals go to a
//                   [blocks, E] histogram;
//   scan kernel     one thread per expert turns the histogram into exclusive
//                   block offsets and yields arrivals, kept counts and the
//                   dropped total;
//   finalize kernel slot = block offset + rank, kept = slot < C, and the
//                   [E, C] row -> token map.
#include <climits>
#include <cmath>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kAssignBlock = 1024;

__device__ __forceinline__ uint64_t splitmix64_at(uint64_t seed, uint64_t t) {
  // output #t of splitmix64 seeded with `seed` (Steele, Lea & Flood 2014)
  uint64_t z = seed + (t + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// logits[t, e] = sum_c x[t, c] * Wr[e, c] + bias[e]   (fp32 FMA chain in c order)
__global__ void router_f32_kernel(int64_t T, int d, int E, const float* __restrict__ x,
                                  const float* __restrict__ Wr, const float* __restrict__ bias,
                                  float* __restrict__ logits) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i >= T * E) return;
  const int64_t t = i / E;
  const int e = static_cast<int>(i - t * E);
  const float* xr = x + t * d;
  const float* wr = Wr + static_cast<int64_t>(e) * d;
  float s = 0.f;
  for (int c = 0; c < d; ++c) s = fmaf(__ldg(xr + c), __ldg(wr + c), s);
  if (bias) s += __ldg(bias + e);
  logits[i] = s;
}

__device__ __forceinline__ bool better(float av, int ai, float bv, int bi) {
  return av > bv || (av == bv && ai < bi);
}

__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    float ov = __shfl_xor_sync(0xffffffffu, v, off);
    int oi = __shfl_xor_sync(0xffffffffu, i, off);
    if (better(ov, oi, v, i)) { v = ov; i = oi; }
  }
}

template <int K>
__global__ void __launch_bounds__(256) gate_topk_kernel(int64_t T, int E,
                                                        const float* __restrict__ logits,
                                                        int32_t* __restrict__ expert_idx,
                                                        float* __restrict__ gate) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t t = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5; t < T;
       t += nwarps) {
    const float* h = logits + t * E;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      v[i] = e < E ? __ldg(h + e) : -INFINITY;
    }
    // best over this lane's experts (ascending index, strict > keeps the lowest on ties)
    float b1v = -INFINITY;
    int b1i = INT_MAX;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (e < E && v[i] > b1v) { b1v = v[i]; b1i = e; }
    }
    warp_argmax(b1v, b1i);
    const float m = b1v;
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (lane + 32 * i < E) s += expf(v[i] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    float b2v = -INFINITY;
    int b2i = INT_MAX;
    if (K == 2) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (e < E && e != b1i && v[i] > b2v) { b2v = v[i]; b2i = e; }
      }
      warp_argmax(b2v, b2i);
    }
    if (lane == 0) {
      expert_idx[t * K] = b1i;
      gate[t * K] = 1.0f / s;  // exp(max - max) / sum
      if (K == 2) {
        expert_idx[t * K + 1] = b2i;
        gate[t * K + 1] = expf(b2v - m) / s;
      }
    }
  }
}

// PanGu-Sigma RRE: expert = domain * (E/G) + splitmix64(seed, t) mod (E/G), gate 1.
__global__ void route_rre_kernel(int64_t T, int E, int G, uint64_t seed,
                                 const int32_t* __restrict__ domain,
                                 int32_t* __restrict__ expert_idx, float* __restrict__ gate,
                                 int32_t* status) {
  const int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (t >= T) return;
  const int per = E / G;
  int dm = __ldg(domain + t);
  if (dm < 0 || dm >= G) {  // out-of-contract id: report, route within group 0
    if (status) atomicOr(status, MOE_STATUS_BAD_DOMAIN);
    dm = 0;
  }
  const uint64_t r = splitmix64_at(seed, static_cast<uint64_t>(t));
  expert_idx[t] = dm * per + static_cast<int>(r % static_cast<uint64_t>(per));
  gate[t] = 1.0f;
}

// rank of each choice among the same expert's choices inside its 1024-block
__global__ void __launch_bounds__(kAssignBlock) assign_rank_kernel(
    int64_t n_assign, int E, const int32_t* __restrict__ expert_idx, int32_t* __restrict__ rank,
    int32_t* __restrict__ block_hist) {
  extern __shared__ int s_cnt[];  // [32 warps][E]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < 32 * E; i += kAssignBlock) s_cnt[i] = 0;
  __syncthreads();
  const int64_t a = static_cast<int64_t>(blockIdx.x) * kAssignBlock + tid;
  int e = a < n_assign ? __ldg(expert_idx + a) : -1;
  if (e >= E) e = -1;
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int r = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && lane == __ffs(peers) - 1) s_cnt[warp * E + e] = __popc(peers);
  __syncthreads();
  for (int x = tid; x < E; x += kAssignBlock) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = s_cnt[w * E + x];
      s_cnt[w * E + x] = run;
      run += c;
    }
    block_hist[static_cast<int64_t>(blockIdx.x) * E + x] = run;
  }
  __syncthreads();
  if (e >= 0) rank[a] = s_cnt[warp * E + e] + r;
}

// per expert: exclusive scan of the block histogram -> block offsets, arrivals, kept, dropped
__global__ void __launch_bounds__(256) assign_scan_kernel(int nblk, int E, int C,
                                                          int32_t* __restrict__ block_hist,
                                                          int32_t* __restrict__ arrivals,
                                                          int32_t* __restrict__ kept_cnt,
                                                          int32_t* __restrict__ n_dropped) {
  __shared__ int s_drop[256];
  int drop = 0;
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int run = 0;
    for (int b = 0; b < nblk; ++b) {
      const int c = block_hist[static_cast<int64_t>(b) * E + x];
      block_hist[static_cast<int64_t>(b) * E + x] = run;
      run += c;
    }
    arrivals[x] = run;
    kept_cnt[x] = run < C ? run : C;
    drop += run > C ? run - C : 0;
  }
  s_drop[threadIdx.x] = drop;
  __syncthreads();
  for (int off = 128; off > 0; off >>= 1) {
    if (threadIdx.x < off) s_drop[threadIdx.x] += s_drop[threadIdx.x + off];
    __syncthreads();
  }
  if (threadIdx.x == 0) n_dropped[0] = s_drop[0];
}

__global__ void __launch_bounds__(256) assign_finalize_kernel(
    int64_t n_assign, int k, int E, int C, const int32_t* __restrict__ expert_idx,
    const int32_t* __restrict__ block_off, int32_t* __restrict__ slot, uint8_t* __restrict__ kept,
    int32_t* __restrict__ tok_of_row, const int32_t* __restrict__ kept_cnt) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i < n_assign) {
    const int e = expert_idx[i];
    if (e >= 0 && e < E) {
      const int s = block_off[(i / kAssignBlock) * E + e] + slot[i];
      slot[i] = s;
      const bool kp = s < C;
      kept[i] = kp ? 1 : 0;
      if (kp) tok_of_row[static_cast<int64_t>(e) * C + s] = static_cast<int32_t>(i / k);
    } else {
      slot[i] = INT_MAX;
      kept[i] = 0;
    }
  }
  if (C > 0 && i < static_cast<int64_t>(E) * C) {
    const int e = static_cast<int>(i / C);
    const int r = static_cast<int>(i - static_cast<int64_t>(e) * C);
    if (r >= kept_cnt[e]) tok_of_row[i] = -1;
  }
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace

size_t assign_scratch_bytes(const moe_config& c) {
  const int64_t n_assign = c.T * c.k;
  return align256(static_cast<size_t>(ceil_div(n_assign, kAssignBlock)) * c.E * sizeof(int32_t));
}

int32_t launch_router_f32(const moe_config& c, const void* x, const void* Wr, const float* bias,
                          float* logits, cudaStream_t s) {
  const int64_t n = c.T * c.E;
  if (n == 0) return MOE_OK;
  router_f32_kernel<<<static_cast<unsigned>(ceil_div(n, 256)), 256, 0, s>>>(
      c.T, c.d_model, c.E, static_cast<const float*>(x), static_cast<const float*>(Wr), bias,
      logits);
  return check_launch("router_f32_kernel");
}

int32_t launch_route_assign(const moe_config& c, const float* logits, const int32_t* domain,
                            int32_t* expert_idx, float* gate, int32_t* slot, uint8_t* kept,
                            int32_t* tok_of_row, int32_t* arrivals, int32_t* kept_cnt,
                            int32_t* n_dropped, void* scratch, int32_t* status, cudaStream_t s) {
  const int64_t T = c.T;
  const int64_t n_assign = T * c.k;
  if (T > 0) {
    if (c.mode == MOE_ROUTE_TOPK) {
      const int64_t blocks = std::min<int64_t>(ceil_div(T, 8), int64_t(num_sms()) * 16);
      if (c.k == 1)
        gate_topk_kernel<1><<<static_cast<unsigned>(blocks), 256, 0, s>>>(T, c.E, logits,
                                                                          expert_idx, gate);
      else
        gate_topk_kernel<2><<<static_cast<unsigned>(blocks), 256, 0, s>>>(T, c.E, logits,
                                                                          expert_idx, gate);
      int32_t rc = check_launch("gate_topk_kernel");
      if (rc != MOE_OK) return rc;
    } else {
      route_rre_kernel<<<static_cast<unsigned>(ceil_div(T, 256)), 256, 0, s>>>(
          T, c.E, c.num_groups, c.seed, domain, expert_idx, gate, status);
      int32_t rc = check_launch("route_rre_kernel");
      if (rc != MOE_OK) return rc;
    }
  }
  int32_t* block_hist = static_cast<int32_t*>(scratch);
  const int64_t nblk = ceil_div(n_assign, kAssignBlock);
  if (nblk > 0) {
    assign_rank_kernel<<<static_cast<unsigned>(nblk), kAssignBlock, 32 * c.E * sizeof(int), s>>>(
        n_assign, c.E, expert_idx, slot, block_hist);
    int32_t rc = check_launch("assign_rank_kernel");
    if (rc != MOE_OK) return rc;
  }
  assign_scan_kernel<<<1, 256, 0, s>>>(static_cast<int>(nblk), c.E, c.capacity, block_hist,
                                       arrivals, kept_cnt, n_dropped);
  int32_t rc = check_launch("assign_scan_kernel");
  if (rc != MOE_OK) return rc;
  const int64_t n_fin = std::max<int64_t>(n_assign, int64_t(c.E) * c.capacity);
  if (n_fin > 0) {
    assign_finalize_kernel<<<static_cast<unsigned>(ceil_div(n_fin, 256)), 256, 0, s>>>(
        n_assign, c.k, c.E, c.capacity, expert_idx, block_hist, slot, kept, tok_of_row, kept_cnt);
    rc = check_launch("assign_finalize_kernel");
  }
  return rc;
}

}  // namespace moe
