// Routing: fp32 router (SIMT), softmax gate + top-k, Random Routed Experts,
// and the capacity-bounded slot assignment.
//
// Gate and top-k (Switch notes sec. 2.1, eq. 1): one warp per token holds the
// token's E <= 256 logits (8 per lane, coalesced), finds the largest with a
// shuffle reduction ordered by (value desc, index asc), the second largest
// the same way with the first excluded, and the softmax denominator
// sum_j exp(h_j - max) with a shuffle sum; gate = exp(h_i - max) / sum.
//
// Slot assignment (sec. 2.2, eq. 3 and the drop rule), in choice order
// (choice a = t*k + j), as ONE kernel on ONE thread-block cluster (16 CTAs
// where the device can co-schedule them, else 8) of 1024 threads each.  The
// cluster's CTAs are resident together by construction, so they exchange
// counts through distributed shared memory with the hardware cluster barrier
// and nothing spins on global flags:
//   1. each warp owns a contiguous run of choices and counts them per expert
//      (__match_any_sync groups the lanes that chose the same expert);
//   2. the 32 warps' counts are prefix-summed per expert in shared memory,
//      giving the CTA's per-expert total; cluster barrier;
//   3. each CTA reads every CTA's totals (DSMEM): the sum over earlier CTAs
//      is its exclusive prefix, the sum over all the arrivals; barrier;
//   4. slot = earlier CTAs + earlier warps + earlier rounds of this warp +
//      rank among this round's peers (the last two kept in registers from
//      step 1 when a warp's run is at most 8 rounds, else found by walking
//      the run again); kept = slot < C, and the row -> token map;
//   5. CTA 0 writes arrivals, kept counts and the dropped total; every CTA
//      marks the free rows of its share of experts with -1.
#include <algorithm>
#include <climits>
#include <cmath>
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kAssignThreads = 1024;
constexpr int kMaxAssignCtas = 16;  // CTAs in the assignment's cluster (16 or 8)
constexpr int kMaxRounds = 8;       // rounds of 32 choices per warp held in registers

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
  dev::pdl_trigger();
  dev::pdl_wait();
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
  dev::pdl_trigger();
  dev::pdl_wait();
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
  dev::pdl_trigger();
  dev::pdl_wait();
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

MOE_DEV int ld_cluster_s32(uint32_t cluster_addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}

struct AssignArgs {
  int64_t n_assign;
  int64_t per_warp;  // choices per warp, a multiple of 32
  int k, E, C;
  const int32_t* expert_idx;
  int32_t* slot;
  uint8_t* kept;
  int32_t* tok_of_row;
  int32_t* arrivals;
  int32_t* kept_cnt;
  int32_t* n_dropped;
};

__global__ void __launch_bounds__(kAssignThreads, 1) assign_kernel(const AssignArgs p) {
  extern __shared__ int s_mem[];
  const int E = p.E;
  // [32 warps][Ep]: counts, then bases for the warp's next round; the odd
  // row stride Ep keeps a column (one expert, all warps) in 32 banks
  const int Ep = E | 1;
  int* s_cnt = s_mem;
  int* s_tot = s_cnt + 32 * Ep;  // [E] this CTA's choices per expert
  int* s_excl = s_tot + E;      // [E] earlier CTAs' choices per expert
  int* s_all = s_excl + E;      // [E] all choices per expert (arrivals)
  __shared__ int s_drop[kAssignThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = static_cast<int>(dev::cta_rank());
  const int nb = static_cast<int>(gridDim.x);  // the grid is one cluster
  const int64_t w0 = (static_cast<int64_t>(b) * (kAssignThreads / 32) + warp) * p.per_warp;
  const int64_t w1 = w0 + p.per_warp < p.n_assign ? w0 + p.per_warp : p.n_assign;
  const unsigned lower = (1u << lane) - 1u;

  dev::pdl_trigger();
  for (int i = tid; i < 32 * Ep; i += kAssignThreads) s_cnt[i] = 0;
  dev::pdl_wait();  // the choices come from the previous kernel
  __syncthreads();

  // 1. this warp's counts per expert (the leader of each group of peers adds).
  //    Runs of up to kMaxRounds rounds keep each lane's choices and their
  //    offsets within the warp's run in registers for step 4.
  const bool in_regs = p.per_warp <= 32 * kMaxRounds;  // the same for every warp
  int ev[kMaxRounds], lv[kMaxRounds];
  if (in_regs) {
#pragma unroll
    for (int r = 0; r < kMaxRounds; ++r) {  // all loads first
      const int64_t a = w0 + 32 * r + lane;
      ev[r] = a < w1 ? __ldg(p.expert_idx + a) : -1;
      if (ev[r] < 0 || ev[r] >= E) ev[r] = -1;
    }
#pragma unroll
    for (int r = 0; r < kMaxRounds; ++r) {
      lv[r] = 0;
      if (w0 + 32 * r < w1) {  // the same for the whole warp
        const int e = ev[r];
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int base = e >= 0 ? s_cnt[warp * Ep + e] : 0;
        __syncwarp();  // every peer has read the base before the leader moves it
        if (e >= 0 && lane == __ffs(peers) - 1) s_cnt[warp * Ep + e] = base + __popc(peers);
        __syncwarp();
        lv[r] = base + __popc(peers & lower);
      }
    }
  } else {
#pragma unroll 4
    for (int64_t base = w0; base < w1; base += 32) {
      const int64_t a = base + lane;
      int e = a < w1 ? __ldg(p.expert_idx + a) : -1;
      if (e < 0 || e >= E) e = -1;
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      if (e >= 0 && lane == __ffs(peers) - 1) s_cnt[warp * Ep + e] += __popc(peers);
      __syncwarp();  // the next round's leader may be another lane
    }
  }
  __syncthreads();
  // 2. exclusive prefix over the warps (choice order), CTA totals: a warp per
  //    expert, lane w holding warp w's count, scanned with shuffles
  for (int x = warp; x < E; x += kAssignThreads / 32) {
    const int c = s_cnt[lane * Ep + x];
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    s_cnt[lane * Ep + x] = incl - c;
    if (lane == 31) s_tot[x] = incl;
  }
  dev::cluster_sync();  // every CTA's totals are final and visible in the cluster
  // 3. earlier CTAs' totals (the exclusive prefix) and all CTAs' (the arrivals):
  //    the cluster's (at most 16) remote loads issued before any is summed
  for (int x = tid; x < E; x += kAssignThreads) {
    const uint32_t addr = dev::smem_u32(s_tot + x);
    int v[kMaxAssignCtas];
#pragma unroll
    for (int q = 0; q < kMaxAssignCtas; ++q) {
      v[q] = 0;
      if (q < nb) {
        uint32_t remote;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(addr), "r"(q));
        v[q] = ld_cluster_s32(remote);
      }
    }
    int before = 0, all = 0;
#pragma unroll
    for (int q = 0; q < kMaxAssignCtas; ++q) {
      before += q < b ? v[q] : 0;
      all += v[q];
    }
    s_excl[x] = before;
    s_all[x] = all;
  }
  dev::cluster_sync();  // no CTA reads another's shared memory after this (it may exit)

  // 4. slots in choice order
  if (in_regs) {
#pragma unroll
    for (int r = 0; r < kMaxRounds; ++r) {
      const int64_t a = w0 + 32 * r + lane;
      if (a < w1) {
        const int e = ev[r];
        const int s = e >= 0 ? s_excl[e] + s_cnt[warp * Ep + e] + lv[r] : INT_MAX;
        p.slot[a] = s;  // INT_MAX for an expert index outside [0, E)
        const bool kp = e >= 0 && s < p.C;
        p.kept[a] = kp ? 1 : 0;
        if (kp) p.tok_of_row[static_cast<int64_t>(e) * p.C + s] = static_cast<int32_t>(a / p.k);
      }
    }
  }
#pragma unroll 4
  for (int64_t base = in_regs ? w1 : w0; base < w1; base += 32) {
    const int64_t a = base + lane;
    const bool in = a < w1;
    int e = in ? __ldg(p.expert_idx + a) : -1;
    if (e < 0 || e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    int s = INT_MAX;
    if (e >= 0) s = s_excl[e] + s_cnt[warp * Ep + e] + __popc(peers & lower);
    __syncwarp();  // every peer has read the base before the leader moves it
    if (e >= 0 && lane == __ffs(peers) - 1) s_cnt[warp * Ep + e] += __popc(peers);
    __syncwarp();
    if (in) {
      p.slot[a] = s;  // INT_MAX for an expert index outside [0, E)
      const bool kp = e >= 0 && s < p.C;
      p.kept[a] = kp ? 1 : 0;
      if (kp) p.tok_of_row[static_cast<int64_t>(e) * p.C + s] = static_cast<int32_t>(a / p.k);
    }
  }

  // 5. totals (CTA 0) and the free rows of the map (experts x = b mod nb, a warp each)
  if (b == 0) {
    int drop = 0;
    for (int x = tid; x < E; x += kAssignThreads) {
      const int arr = s_all[x];
      const int kc = arr < p.C ? arr : p.C;
      p.arrivals[x] = arr;
      p.kept_cnt[x] = kc;
      drop += arr - kc;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) drop += __shfl_xor_sync(0xffffffffu, drop, off);
    if (lane == 0) s_drop[warp] = drop;
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < kAssignThreads / 32; ++w) tot += s_drop[w];
      p.n_dropped[0] = tot;
    }
  }
  for (int x = b + nb * warp; x < E; x += nb * (kAssignThreads / 32)) {
    const int kc = s_all[x] < p.C ? s_all[x] : p.C;
    for (int r = kc + lane; r < p.C; r += 32)
      p.tok_of_row[static_cast<int64_t>(x) * p.C + r] = -1;
  }
}

// Totals for a call with no choices (T = 0): zero counts, empty row map.
__global__ void assign_empty_kernel(int E, int C, int32_t* arrivals, int32_t* kept_cnt,
                                    int32_t* n_dropped, int32_t* tok_of_row) {
  dev::pdl_trigger();
  dev::pdl_wait();
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    arrivals[x] = 0;
    kept_cnt[x] = 0;
  }
  if (threadIdx.x == 0) n_dropped[0] = 0;
  const int64_t rows = static_cast<int64_t>(E) * C;
  for (int64_t i = threadIdx.x; i < rows; i += blockDim.x) tok_of_row[i] = -1;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace

// The assignment needs no global scratch (its CTAs exchange counts in
// distributed shared memory).
size_t assign_scratch_bytes(const moe_config&) { return 0; }

int32_t launch_router_f32(const moe_config& c, const void* x, const void* Wr, const float* bias,
                          float* logits, cudaStream_t s) {
  const int64_t n = c.T * c.E;
  if (n == 0) return MOE_OK;
  launch_pdl(router_f32_kernel, dim3(static_cast<unsigned>(ceil_div(n, 256))), dim3(256), 0, s,
             c.T, c.d_model, c.E, static_cast<const float*>(x), static_cast<const float*>(Wr),
             bias, logits);
  return check_launch("router_f32_kernel");
}

int32_t launch_route_assign(const moe_config& c, const float* logits, const int32_t* domain,
                            int32_t* expert_idx, float* gate, int32_t* slot, uint8_t* kept,
                            int32_t* tok_of_row, int32_t* arrivals, int32_t* kept_cnt,
                            int32_t* n_dropped, void* scratch, int32_t* status, cudaStream_t s) {
  const int64_t T = c.T;
  if (T > 0) {
    if (c.mode == MOE_ROUTE_TOPK) {
      const int64_t blocks = std::min<int64_t>(ceil_div(T, 8), int64_t(num_sms()) * 16);
      if (c.k == 1)
        launch_pdl(gate_topk_kernel<1>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, T,
                   c.E, logits, expert_idx, gate);
      else
        launch_pdl(gate_topk_kernel<2>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, T,
                   c.E, logits, expert_idx, gate);
      int32_t rc = check_launch("gate_topk_kernel");
      if (rc != MOE_OK) return rc;
    } else {
      launch_pdl(route_rre_kernel, dim3(static_cast<unsigned>(ceil_div(T, 256))), dim3(256), 0, s,
                 T, c.E, c.num_groups, c.seed, domain, expert_idx, gate, status);
      int32_t rc = check_launch("route_rre_kernel");
      if (rc != MOE_OK) return rc;
    }
  }
  return launch_assign(c, expert_idx, slot, kept, tok_of_row, arrivals, kept_cnt, n_dropped,
                       scratch, status, s);
}

namespace {

size_t assign_smem_bytes(int E) { return (32 * static_cast<size_t>(E | 1) + 3 * E) * sizeof(int); }

// CTAs in the assignment's cluster: 16 where the device co-schedules a
// cluster of 16 such CTAs (a non-portable size), else the portable 8.
// Queried once per device.
int32_t assign_cluster_size(int* out) {
  constexpr int kMaxDev = 64;
  static int cache[kMaxDev] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return check_launch("cudaGetDevice");
  std::lock_guard<std::mutex> lock(mu);
  if (dev < kMaxDev && cache[dev] > 0) {
    *out = cache[dev];
    return MOE_OK;
  }
  const size_t smem = assign_smem_bytes(256);
  if (cudaFuncSetAttribute(assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess ||
      cudaFuncSetAttribute(assign_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
          cudaSuccess)
    return check_launch("cudaFuncSetAttribute(assign_kernel)");
  int size = 8;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(16);
  cfg.blockDim = dim3(kAssignThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 16;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, assign_kernel, &cfg) == cudaSuccess && clusters >= 1)
    size = 16;
  cudaGetLastError();  // a refused query leaves no error behind
  if (dev < kMaxDev) cache[dev] = size;
  *out = size;
  return MOE_OK;
}

}  // namespace

// The slot assignment alone, from the choices expert_idx [T, k] written
// earlier on the same stream.
int32_t launch_assign(const moe_config& c, const int32_t* expert_idx, int32_t* slot,
                      uint8_t* kept, int32_t* tok_of_row, int32_t* arrivals, int32_t* kept_cnt,
                      int32_t* n_dropped, void* scratch, int32_t* status, cudaStream_t s) {
  (void)scratch;
  (void)status;
  const int64_t n_assign = c.T * c.k;
  if (n_assign == 0) {
    launch_pdl(assign_empty_kernel, dim3(1), dim3(256), 0, s, c.E, c.capacity, arrivals, kept_cnt,
               n_dropped, tok_of_row);
    return check_launch("assign_empty_kernel");
  }
  int nb = 0;
  int32_t rc = assign_cluster_size(&nb);
  if (rc != MOE_OK) return rc;
  AssignArgs p{};
  p.n_assign = n_assign;
  // choices per warp: the whole list over nb * 32 warps, in rounds of 32
  p.per_warp = ceil_div(ceil_div(n_assign, int64_t(nb) * (kAssignThreads / 32)), 32) * 32;
  p.k = c.k;
  p.E = c.E;
  p.C = c.capacity;
  p.expert_idx = expert_idx;
  p.slot = slot;
  p.kept = kept;
  p.tok_of_row = tok_of_row;
  p.arrivals = arrivals;
  p.kept_cnt = kept_cnt;
  p.n_dropped = n_dropped;
  // on every launch: a function attribute belongs to the current context, the
  // cached cluster size to the device
  if (cudaFuncSetAttribute(assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(assign_smem_bytes(256))) != cudaSuccess ||
      cudaFuncSetAttribute(assign_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
          cudaSuccess)
    return check_launch("cudaFuncSetAttribute(assign_kernel)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(nb));
  cfg.blockDim = dim3(kAssignThreads);
  cfg.dynamicSmemBytes = assign_smem_bytes(c.E);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(nb);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaLaunchKernelEx(&cfg, assign_kernel, p);
  return check_launch("assign_kernel");
}

}  // namespace moe
