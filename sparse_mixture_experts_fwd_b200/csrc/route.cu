// Routing: fp32 router (SIMT), softmax gate + top-k, Random Routed Experts,
// and the capacity-bounded slot assignment.
//
// Gate and top-k (Switch notes sec. 2.1, eq. 1): one warp per token holds the
// token's E <= 256 logits (8 per lane, coalesced), finds the largest with a
// shuffle reduction ordered by (value desc, index asc), the second largest
// the same way with the first excluded, and the softmax denominator
// sum_j exp(h_j - max) with a shuffle sum; gate = exp(h_i - max) / sum.
//
// Slot assignment (sec. 2.2, eq. 3 and the drop rule), in token order, as ONE
// kernel over blocks of 1024 choices (choice a = t*k + j):
//   1. rank inside the block: __match_any_sync groups the lanes that chose
//      the same expert, __popc of the lower peers gives the rank inside the
//      warp, per-warp counts are prefix-summed in shared memory across the 32
//      warps; the block's per-expert counts are its aggregate;
//   2. decoupled look-back: the block publishes its aggregate (flag 1), reads
//      the flags of all earlier blocks, and sums their aggregates back to the
//      nearest block that already published its inclusive prefix (flag 2),
//      then publishes its own inclusive prefix (flag 2);
//   3. slot = exclusive prefix + rank, kept = slot < C, row -> token map;
//      the last block also writes arrivals, kept counts, the dropped total
//      and marks free rows of the map with -1.
// The flags are cleared by the kernel that produced the choices (stream
// order), and every wait on a flag is bounded by time.
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

__device__ __forceinline__ void clear_flags(unsigned int* flags, int nblk) {
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < nblk; i += blockDim.x) flags[i] = 0u;
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
                                                        float* __restrict__ gate,
                                                        unsigned int* flags, int nblk) {
  dev::pdl_trigger();
  dev::pdl_wait();
  clear_flags(flags, nblk);
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
                                 int32_t* status, unsigned int* flags, int nblk) {
  dev::pdl_trigger();
  dev::pdl_wait();
  clear_flags(flags, nblk);
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

MOE_DEV unsigned int ld_acquire(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
MOE_DEV void st_release(unsigned int* p, unsigned int v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

struct AssignArgs {
  int64_t n_assign;
  int k, E, C, nblk;
  const int32_t* expert_idx;
  int32_t* slot;
  uint8_t* kept;
  int32_t* tok_of_row;
  int32_t* arrivals;
  int32_t* kept_cnt;
  int32_t* n_dropped;
  unsigned int* flags;  // [nblk], cleared before launch
  int32_t* aggr;        // [nblk][E]
  int32_t* incl;        // [nblk][E]
  int32_t* status;      // nullable; also the call's give-up signal
  uint64_t wait_ns;     // limit of the look-back wait
};

__global__ void __launch_bounds__(kAssignBlock, 1) assign_kernel(const AssignArgs p) {
  extern __shared__ int s_cnt[];  // [32 warps][E], then excl[E]
  __shared__ int s_pstar, s_ok, s_maxinc, s_maxbad, s_drop[32], s_ticket;
  int* s_excl = s_cnt + 32 * p.E;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = p.E;

  // 1. ranks inside the block
  dev::pdl_trigger();
  for (int i = tid; i < 32 * E; i += kAssignBlock) s_cnt[i] = 0;
  dev::pdl_wait();
  // The block's place in token order is a ticket taken when it starts, not
  // blockIdx: a block then only ever waits on blocks that are already running,
  // whatever order the hardware starts them in.
  if (tid == 0) s_ticket = static_cast<int>(atomicAdd(p.flags + p.nblk, 1u));
  __syncthreads();
  const int b = s_ticket;
  const int64_t a = static_cast<int64_t>(b) * kAssignBlock + tid;
  int e = a < p.n_assign ? __ldg(p.expert_idx + a) : -1;
  if (e >= E) e = -1;
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int r_in_warp = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && lane == __ffs(peers) - 1) s_cnt[warp * E + e] = __popc(peers);
  __syncthreads();
  for (int x = tid; x < E; x += kAssignBlock) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = s_cnt[w * E + x];
      s_cnt[w * E + x] = run;
      run += c;
    }
    p.aggr[static_cast<int64_t>(b) * E + x] = run;  // block aggregate
    s_excl[x] = 0;
    if (b == 0) p.incl[x] = run;
  }
  // 2. publish the aggregate (or, for block 0, the inclusive prefix)
  __threadfence();
  __syncthreads();
  if (tid == 0) st_release(p.flags + b, b == 0 ? 2u : 1u);

  if (b > 0) {
    // p*: the latest earlier block with an inclusive prefix, usable once every
    // block after it has at least published its aggregate.  All earlier flags
    // are read in parallel (one thread each) and reduced in shared memory.
    const unsigned long long t0 = dev::globaltimer();
    for (;;) {
      if (tid == 0) {
        s_maxinc = -1;
        s_maxbad = -1;
      }
      __syncthreads();
      for (int q = tid; q < b; q += kAssignBlock) {
        const unsigned int f = ld_acquire(p.flags + q);
        if (f == 2u) atomicMax(&s_maxinc, q);
        else if (f == 0u) atomicMax(&s_maxbad, q);
      }
      __syncthreads();
      const bool ready = s_maxinc >= 0 && s_maxbad < s_maxinc;
      if (tid == 0) {
        s_pstar = s_maxinc;
        if (ready) {
          s_ok = 1;
        } else if (p.status &&
                   (*reinterpret_cast<volatile int32_t*>(p.status) & MOE_STATUS_TIMEOUT)) {
          s_ok = -1;  // another wait of this call has already given up
        } else if (dev::globaltimer() - t0 > p.wait_ns) {
          s_ok = -1;
          if (p.status) atomicOr(p.status, MOE_STATUS_TIMEOUT);
        } else {
          s_ok = 0;
        }
      }
      __syncthreads();
      if (s_ok != 0) break;
    }
    if (s_ok < 0) return;  // bounded wait expired: outputs are invalid, status says so
    const int pstar = s_pstar;
    for (int x = tid; x < E; x += kAssignBlock) {
      // the aggregates after p* are independent loads: 8 in flight per round
      int acc = __ldcg(p.incl + static_cast<int64_t>(pstar) * E + x);
      int part[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      int q = pstar + 1;
      for (; q + 8 <= b; q += 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) part[u] += __ldcg(p.aggr + static_cast<int64_t>(q + u) * E + x);
      }
      for (; q < b; ++q) part[0] += __ldcg(p.aggr + static_cast<int64_t>(q) * E + x);
#pragma unroll
      for (int u = 0; u < 8; ++u) acc += part[u];
      s_excl[x] = acc;
      p.incl[static_cast<int64_t>(b) * E + x] = acc + p.aggr[static_cast<int64_t>(b) * E + x];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release(p.flags + b, 2u);
  } else {
    __syncthreads();
  }

  // 3. slots, kept mask, row -> token map
  if (a < p.n_assign) {
    if (e >= 0) {
      const int s = s_excl[e] + s_cnt[warp * E + e] + r_in_warp;
      p.slot[a] = s;
      const bool kp = s < p.C;
      p.kept[a] = kp ? 1 : 0;
      if (kp) p.tok_of_row[static_cast<int64_t>(e) * p.C + s] = static_cast<int32_t>(a / p.k);
    } else {
      p.slot[a] = INT_MAX;
      p.kept[a] = 0;
    }
  }
  // the last block owns the totals
  if (b == p.nblk - 1) {
    __syncthreads();  // every thread is done reading the rank table reused below
    int drop = 0;
    for (int x = tid; x < E; x += kAssignBlock) {
      const int arr = s_excl[x] + p.aggr[static_cast<int64_t>(b) * E + x];
      p.arrivals[x] = arr;
      const int kc = arr < p.C ? arr : p.C;
      p.kept_cnt[x] = kc;
      s_cnt[x] = kc;  // reuse: kept count per expert for the -1 fill below
      drop += arr - kc;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) drop += __shfl_xor_sync(0xffffffffu, drop, off);
    if (lane == 0) s_drop[warp] = drop;
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < 32; ++w) tot += s_drop[w];
      p.n_dropped[0] = tot;
    }
    // free rows of the map: a warp per expert, lanes over its rows past the kept count
    for (int ex = warp; ex < E; ex += kAssignBlock / 32)
      for (int r = s_cnt[ex] + lane; r < p.C; r += 32)
        p.tok_of_row[static_cast<int64_t>(ex) * p.C + r] = -1;
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

// the look-back flags [nblk] and the block ticket counter after them
int assign_flag_words(const moe_config& c) {
  return static_cast<int>(ceil_div(c.T * c.k, kAssignBlock)) + 1;
}

// flags [nblk] u32 + ticket u32, then aggr and incl [nblk][E] i32 each
size_t assign_scratch_bytes(const moe_config& c) {
  const int64_t nblk = ceil_div(c.T * c.k, kAssignBlock);
  return align256(static_cast<size_t>(nblk + 1) * sizeof(unsigned int)) +
         2 * align256(static_cast<size_t>(nblk) * c.E * sizeof(int32_t));
}

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
  const int64_t n_assign = T * c.k;
  const int64_t nblk = ceil_div(n_assign, kAssignBlock);
  char* sc = static_cast<char*>(scratch);
  unsigned int* flags = reinterpret_cast<unsigned int*>(sc);
  const size_t flags_bytes = align256(static_cast<size_t>(nblk + 1) * sizeof(unsigned int));
  const size_t vec_bytes = align256(static_cast<size_t>(nblk) * c.E * sizeof(int32_t));
  int32_t* aggr = reinterpret_cast<int32_t*>(sc + flags_bytes);
  int32_t* incl = reinterpret_cast<int32_t*>(sc + flags_bytes + vec_bytes);
  if (T == 0) {
    launch_pdl(assign_empty_kernel, dim3(1), dim3(256), 0, s, c.E, c.capacity, arrivals, kept_cnt, n_dropped,
                                          tok_of_row);
    return check_launch("assign_empty_kernel");
  }
  if (c.mode == MOE_ROUTE_TOPK) {
    const int64_t blocks = std::min<int64_t>(ceil_div(T, 8), int64_t(num_sms()) * 16);
    if (c.k == 1)
      launch_pdl(gate_topk_kernel<1>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, T,
                 c.E, logits, expert_idx, gate, flags, static_cast<int>(nblk + 1));
    else
      launch_pdl(gate_topk_kernel<2>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, T,
                 c.E, logits, expert_idx, gate, flags, static_cast<int>(nblk + 1));
    int32_t rc = check_launch("gate_topk_kernel");
    if (rc != MOE_OK) return rc;
  } else {
    launch_pdl(route_rre_kernel, dim3(static_cast<unsigned>(ceil_div(T, 256))), dim3(256), 0, s,
               T, c.E, c.num_groups, c.seed, domain, expert_idx, gate, status, flags,
               static_cast<int>(nblk + 1));
    int32_t rc = check_launch("route_rre_kernel");
    if (rc != MOE_OK) return rc;
  }
  return launch_assign(c, expert_idx, slot, kept, tok_of_row, arrivals, kept_cnt, n_dropped,
                       scratch, status, s);
}

// The slot assignment alone, from choices whose look-back flags are already
// cleared (by the kernel that produced them, earlier on the same stream).
int32_t launch_assign(const moe_config& c, const int32_t* expert_idx, int32_t* slot,
                      uint8_t* kept, int32_t* tok_of_row, int32_t* arrivals, int32_t* kept_cnt,
                      int32_t* n_dropped, void* scratch, int32_t* status, cudaStream_t s) {
  const int64_t n_assign = c.T * c.k;
  const int64_t nblk = ceil_div(n_assign, kAssignBlock);
  if (nblk == 0) {
    launch_pdl(assign_empty_kernel, dim3(1), dim3(256), 0, s, c.E, c.capacity, arrivals, kept_cnt, n_dropped,
                                          tok_of_row);
    return check_launch("assign_empty_kernel");
  }
  char* sc = static_cast<char*>(scratch);
  const size_t flags_bytes = align256(static_cast<size_t>(nblk + 1) * sizeof(unsigned int));
  const size_t vec_bytes = align256(static_cast<size_t>(nblk) * c.E * sizeof(int32_t));
  AssignArgs p{};
  p.n_assign = n_assign;
  p.k = c.k;
  p.E = c.E;
  p.C = c.capacity;
  p.nblk = static_cast<int>(nblk);
  p.expert_idx = expert_idx;
  p.slot = slot;
  p.kept = kept;
  p.tok_of_row = tok_of_row;
  p.arrivals = arrivals;
  p.kept_cnt = kept_cnt;
  p.n_dropped = n_dropped;
  p.flags = reinterpret_cast<unsigned int*>(sc);
  p.aggr = reinterpret_cast<int32_t*>(sc + flags_bytes);
  p.incl = reinterpret_cast<int32_t*>(sc + flags_bytes + vec_bytes);
  p.status = status;
  p.wait_ns = wait_limit_ns();
  const size_t smem = (33 * static_cast<size_t>(c.E)) * sizeof(int);
  launch_pdl(assign_kernel, dim3(static_cast<unsigned>(nblk)), dim3(kAssignBlock), smem, s, p);
  return check_launch("assign_kernel");
}

}  // namespace moe
