// Dispatch and combine: the two HBM-bound permutations around the experts.
//
// Dispatch (the row permutation behind the Switch router's dispatch tensor,
// Switch notes sec. 2.4): a warp owns one token, reads its row of x once with
// 16-byte loads and writes it to the expert slot of every kept choice, so a
// dropped token costs no activation traffic at all.
//
// Combine (sec. 2.1 eq. 2, drop rule sec. 2.2): a warp owns one token,
// gathers the k expert output rows with 16-byte loads, accumulates
// gate * row in fp32 (choice order j = 0, 1) and writes the token's row once,
// rounded to the activation type; a token with no kept choice gets zeros.
//
// Expert-parallel forms (Switch notes sec. 2, opening: the sparse layer's
// distinct expert weights live on different devices, so the parameter count
// grows with the device count): `world` ranks, rank r holds experts
// r*El .. (r+1)*El - 1 and routes its own batch.  Expert e's rows on its home
// rank h = e / El form one [world*C, d] block of the receive buffer
// [El, world*C, d]; the rows from rank q start at off_q(e) = sum over q' < q
// of q''s kept count of e, in q's slot (token) order.  ep_dispatch_kernel
// stores each kept row straight into the home rank's buffer through its peer
// mapping (NVLink stores; a plain store when h is this rank), and
// ep_combine_kernel loads each token's expert outputs back the same way.  A
// one-thread ep_release_kernel after the dispatch issues the single
// system-scope fence that publishes the copy's peer stores.  None of them
// waits on another rank: the caller orders dispatch -> expert FFN -> combine
// across ranks (a collective between the steps).
#include <algorithm>

#include "moe_internal.cuh"

namespace moe {
namespace {

// A kept choice's expert and slot inside [0, E) x [0, C).  The bounds-checked
// build tests them before a row is touched; the default build trusts them.
__device__ __forceinline__ bool choice_in_range(int e, int s, int E, int C) {
#if MOE_CHECK_BOUNDS
  return e >= 0 && e < E && s >= 0 && s < C;
#else
  (void)e; (void)s; (void)E; (void)C;
  return true;
#endif
}

template <int K>
__global__ void __launch_bounds__(256) dispatch_kernel(int64_t T, int row_vec, int E, int C,
                                                       const uint4* __restrict__ x,
                                                       const int32_t* __restrict__ expert_idx,
                                                       const int32_t* __restrict__ slot,
                                                       const uint8_t* __restrict__ kept,
                                                       uint4* __restrict__ xe,
                                                       unsigned int* __restrict__ zero_words,
                                                       int n_zero, uint4* __restrict__ y_zero,
                                                       int32_t* __restrict__ status) {
  dev::pdl_trigger();
  dev::pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  // counters the next kernel on this stream expects at zero (the fused expert FFN)
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero_words[i] = 0u;
  bool bad = false;
  for (int64_t t = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5; t < T;
       t += nwarps) {
    int64_t dst0 = 0, dst1 = 0;  // the kept choices' xe rows, in choice order
    int nd = 0;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      if (__ldg(kept + t * K + j)) {
        const int e = __ldg(expert_idx + t * K + j), sl = __ldg(slot + t * K + j);
        if (!choice_in_range(e, sl, E, C)) {
          bad = true;
          continue;
        }
        const int64_t d = (static_cast<int64_t>(e) * C + sl) * row_vec;
        if (nd == 0) dst0 = d;
        else dst1 = d;
        ++nd;
      }
    }
    if (nd == 0) {
      // top-1 layers combine inside the expert FFN, which writes only kept
      // tokens; a dropped token's output row is 0 (drop rule)
      if (y_zero)
        for (int v = lane; v < row_vec; v += 32) y_zero[t * row_vec + v] = make_uint4(0, 0, 0, 0);
      continue;
    }
    const uint4* src = x + t * row_vec;
#pragma unroll 4
    for (int v = lane; v < row_vec; v += 32) {
      const uint4 val = __ldg(src + v);
      xe[dst0 + v] = val;
      if (K == 2 && nd == 2) xe[dst1 + v] = val;
    }
  }
  if (MOE_CHECK_BOUNDS && bad && lane == 0 && status) atomicOr(status, MOE_STATUS_BAD_INDEX);
}

struct Bf16x8 {
  static constexpr int kN = 8;
  static __device__ __forceinline__ void unpack(const uint4& u, float (&f)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 p = __bfloat1622float2(h[i]);
      f[2 * i] = p.x;
      f[2 * i + 1] = p.y;
    }
  }
  static __device__ __forceinline__ uint4 pack(const float (&f)[8]) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return u;
  }
};

struct F32x4 {
  static constexpr int kN = 4;
  static __device__ __forceinline__ void unpack(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
  static __device__ __forceinline__ uint4 pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

template <int K, class V>
__global__ void __launch_bounds__(256) combine_kernel(int64_t T, int row_vec, int E, int C,
                                                      const uint4* __restrict__ ye,
                                                      const int32_t* __restrict__ expert_idx,
                                                      const float* __restrict__ gate,
                                                      const int32_t* __restrict__ slot,
                                                      const uint8_t* __restrict__ kept,
                                                      uint4* __restrict__ y,
                                                      int32_t* __restrict__ status) {
  dev::pdl_trigger();
  dev::pdl_wait();
  constexpr int N = V::kN;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  bool bad = false;
  for (int64_t t = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5; t < T;
       t += nwarps) {
    int64_t src[K];
    float g[K];
    int ns = 0;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      if (__ldg(kept + t * K + j)) {
        const int e = __ldg(expert_idx + t * K + j), sl = __ldg(slot + t * K + j);
        if (!choice_in_range(e, sl, E, C)) {
          bad = true;
          continue;
        }
        src[ns] = (static_cast<int64_t>(e) * C + sl) * row_vec;
        g[ns] = __ldg(gate + t * K + j);
        ++ns;
      }
    }
    uint4* dst = y + t * row_vec;
#pragma unroll 2
    for (int v = lane; v < row_vec; v += 32) {
      float acc[N];
#pragma unroll
      for (int i = 0; i < N; ++i) acc[i] = 0.f;
      if (ns > 0) {
        uint4 r0 = __ldg(ye + src[0] + v);
        uint4 r1 = make_uint4(0, 0, 0, 0);
        if (K == 2 && ns == 2) r1 = __ldg(ye + src[K - 1] + v);
        float f[N];
        V::unpack(r0, f);
#pragma unroll
        for (int i = 0; i < N; ++i) acc[i] = g[0] * f[i];
        if (K == 2 && ns == 2) {
          V::unpack(r1, f);
#pragma unroll
          for (int i = 0; i < N; ++i) acc[i] = fmaf(g[K - 1], f[i], acc[i]);
        }
      }
      dst[v] = V::pack(acc);
    }
  }
  if (MOE_CHECK_BOUNDS && bad && lane == 0 && status) atomicOr(status, MOE_STATUS_BAD_INDEX);
}

unsigned grid_for_tokens(int64_t T) {
  const int64_t want = (T + 7) / 8;  // 8 warps per block, a warp per token
  return static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(want, int64_t(num_sms()) * 16)));
}

// peer buffers of the ranks of one node, by rank
struct PeerRows {
  uint4* p[kMaxEpRanks];
};
struct PeerRowsConst {
  const uint4* p[kMaxEpRanks];
};

// entry h of a kernel-parameter table, by selects (a dynamic index would copy
// the table to local memory)
template <class P>
__device__ __forceinline__ auto pick(const P& t, int h) -> decltype(t.p[0]) {
  auto r = t.p[0];
#pragma unroll
  for (int q = 1; q < kMaxEpRanks; ++q)
    if (h == q) r = t.p[q];
  return r;
}

// off[e] = rows of expert e that ranks 0..rank-1 send ahead of this rank's
__device__ __forceinline__ void ep_offsets(const int32_t* __restrict__ cnt_all, int E, int rank,
                                           int* off) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int o = 0;
    for (int q = 0; q < rank; ++q) o += __ldg(cnt_all + static_cast<int64_t>(q) * E + e);
    off[e] = o;
  }
}

template <int K>
__global__ void __launch_bounds__(256) ep_dispatch_kernel(
    int64_t T, int row_vec, int E, int El, int rank, int world, int PC, const uint4* __restrict__ x,
    const int32_t* __restrict__ expert_idx, const int32_t* __restrict__ slot,
    const uint8_t* __restrict__ kept, const int32_t* __restrict__ cnt_all, PeerRows xe,
    int32_t* __restrict__ local_cnt, int32_t* __restrict__ status) {
  __shared__ int s_off[256];
  dev::pdl_trigger();
  dev::pdl_wait();
  ep_offsets(cnt_all, E, rank, s_off);
  // rows each of this rank's experts receives from all ranks (the FFN's counts)
  if (blockIdx.x == 0 && local_cnt)
    for (int el = threadIdx.x; el < El; el += blockDim.x) {
      int n = 0;
      for (int q = 0; q < world; ++q)
        n += __ldg(cnt_all + static_cast<int64_t>(q) * E + static_cast<int64_t>(rank) * El + el);
      local_cnt[el] = n;
    }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  bool bad = false;
  for (int64_t t = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5; t < T;
       t += nwarps) {
    uint4* dst0 = nullptr;  // the kept choices' destination rows, in choice order
    uint4* dst1 = nullptr;
    int nd = 0;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      if (!__ldg(kept + t * K + j)) continue;
      const int e = __ldg(expert_idx + t * K + j);
      const int64_t row = int64_t(e >= 0 && e < E ? s_off[e] : -1) + __ldg(slot + t * K + j);
      if (e < 0 || e >= E || row < 0 || row >= PC) {  // counts that do not match the assignment
        bad = true;
        continue;
      }
      const int h = e / El;
      uint4* d = pick(xe, h) + (static_cast<int64_t>(e - h * El) * PC + row) * row_vec;
      if (nd == 0) dst0 = d;
      else dst1 = d;
      ++nd;
    }
    if (nd == 0) continue;
    const uint4* src = x + t * row_vec;
#pragma unroll 4
    for (int v = lane; v < row_vec; v += 32) {
      const uint4 val = __ldg(src + v);
      dst0[v] = val;
      if (K == 2 && nd == 2) dst1[v] = val;
    }
  }
  if (bad && lane == 0 && status) atomicOr(status, MOE_STATUS_BAD_COUNTS);
}

// Runs after ep_dispatch_kernel on the same stream: griddepcontrol.wait
// returns once the dispatch grid has completed and its stores are visible to
// this grid, and the system-scope fence (cumulative over what this thread has
// observed) then makes them visible to every device before the caller's next
// operation, the cross-rank barrier.  One fence per dispatch instead of one
// per warp, which would hold every warp of the copy until its peer stores are
// acknowledged.
__global__ void __launch_bounds__(32) ep_release_kernel() {
  dev::pdl_trigger();
  dev::pdl_wait();
  if (threadIdx.x == 0) __threadfence_system();
}

template <int K, class V>
__global__ void __launch_bounds__(256) ep_combine_kernel(
    int64_t T, int row_vec, int E, int El, int rank, int PC, PeerRowsConst ye,
    const int32_t* __restrict__ expert_idx, const float* __restrict__ gate,
    const int32_t* __restrict__ slot, const uint8_t* __restrict__ kept,
    const int32_t* __restrict__ cnt_all, uint4* __restrict__ y, int32_t* __restrict__ status) {
  __shared__ int s_off[256];
  dev::pdl_trigger();
  dev::pdl_wait();
  ep_offsets(cnt_all, E, rank, s_off);
  __syncthreads();
  constexpr int N = V::kN;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  bool bad = false;
  for (int64_t t = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5; t < T;
       t += nwarps) {
    const uint4* src0 = nullptr;  // the kept choices' rows and gates, in choice order
    const uint4* src1 = nullptr;
    float g0 = 0.f, g1 = 0.f;
    int ns = 0;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      if (!__ldg(kept + t * K + j)) continue;
      const int e = __ldg(expert_idx + t * K + j);
      const int64_t row = int64_t(e >= 0 && e < E ? s_off[e] : -1) + __ldg(slot + t * K + j);
      if (e < 0 || e >= E || row < 0 || row >= PC) {
        bad = true;
        continue;
      }
      const int h = e / El;
      const uint4* r = pick(ye, h) + (static_cast<int64_t>(e - h * El) * PC + row) * row_vec;
      const float gj = __ldg(gate + t * K + j);
      if (ns == 0) {
        src0 = r;
        g0 = gj;
      } else {
        src1 = r;
        g1 = gj;
      }
      ++ns;
    }
    uint4* dst = y + t * row_vec;
#pragma unroll 2
    for (int v = lane; v < row_vec; v += 32) {
      float acc[N];
#pragma unroll
      for (int i = 0; i < N; ++i) acc[i] = 0.f;
      if (ns > 0) {
        const uint4 r0 = __ldg(src0 + v);
        uint4 r1 = make_uint4(0, 0, 0, 0);
        if (K == 2 && ns == 2) r1 = __ldg(src1 + v);
        float f[N];
        V::unpack(r0, f);
#pragma unroll
        for (int i = 0; i < N; ++i) acc[i] = g0 * f[i];
        if (K == 2 && ns == 2) {
          V::unpack(r1, f);
#pragma unroll
          for (int i = 0; i < N; ++i) acc[i] = fmaf(g1, f[i], acc[i]);
        }
      }
      dst[v] = V::pack(acc);
    }
  }
  if (bad && lane == 0 && status) atomicOr(status, MOE_STATUS_BAD_COUNTS);
}

}  // namespace

int32_t launch_dispatch(const moe_config& c, const void* x, const int32_t* expert_idx,
                        const int32_t* slot, const uint8_t* kept, void* xe, int32_t* status,
                        cudaStream_t s, unsigned int* zero_words, int n_zero, void* y_zero) {
  if (c.T == 0 || (c.capacity == 0 && !y_zero)) return MOE_OK;
  const int row_vec = static_cast<int>(c.d_model * elem_size(c.dtype) / 16);
  const unsigned grid = grid_for_tokens(c.T);
  uint4* yz = static_cast<uint4*>(y_zero);
  if (c.k == 1)
    launch_pdl(dispatch_kernel<1>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.E, c.capacity,
               static_cast<const uint4*>(x), expert_idx, slot, kept, static_cast<uint4*>(xe),
               zero_words, n_zero, yz, status);
  else
    launch_pdl(dispatch_kernel<2>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.E, c.capacity,
               static_cast<const uint4*>(x), expert_idx, slot, kept, static_cast<uint4*>(xe),
               zero_words, n_zero, yz, status);
  return check_launch("dispatch_kernel");
}

int32_t launch_combine(const moe_config& c, const void* ye, const int32_t* expert_idx,
                       const float* gate, const int32_t* slot, const uint8_t* kept, void* y,
                       int32_t* status, cudaStream_t s) {
  if (c.T == 0) return MOE_OK;
  const int row_vec = static_cast<int>(c.d_model * elem_size(c.dtype) / 16);
  const unsigned grid = grid_for_tokens(c.T);
  const uint4* yev = static_cast<const uint4*>(ye);
  uint4* yv = static_cast<uint4*>(y);
  if (c.dtype == MOE_DTYPE_BF16) {
    if (c.k == 1)
      launch_pdl(combine_kernel<1, Bf16x8>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.E, c.capacity, yev, expert_idx,
                                                     gate, slot, kept, yv, status);
    else
      launch_pdl(combine_kernel<2, Bf16x8>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.E, c.capacity, yev, expert_idx,
                                                     gate, slot, kept, yv, status);
  } else {
    if (c.k == 1)
      launch_pdl(combine_kernel<1, F32x4>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.E, c.capacity, yev, expert_idx,
                                                    gate, slot, kept, yv, status);
    else
      launch_pdl(combine_kernel<2, F32x4>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.E, c.capacity, yev, expert_idx,
                                                    gate, slot, kept, yv, status);
  }
  return check_launch("combine_kernel");
}

int32_t launch_ep_dispatch(const moe_config& c, int rank, int world, const void* x,
                           const int32_t* expert_idx, const int32_t* slot, const uint8_t* kept,
                           const int32_t* cnt_all, void* const* xe_peers, int32_t* local_cnt,
                           int32_t* status, cudaStream_t s) {
  const int row_vec = static_cast<int>(c.d_model * elem_size(c.dtype) / 16);
  const int El = c.E / world;
  const int PC = world * c.capacity;
  PeerRows xe{};
  for (int q = 0; q < world && xe_peers; ++q) xe.p[q] = static_cast<uint4*>(xe_peers[q]);
  // T = 0 still writes local_cnt (other ranks' rows arrive all the same)
  const unsigned grid = grid_for_tokens(std::max<int64_t>(c.T, 1));
  const uint4* xv = static_cast<const uint4*>(x);
  if (c.k == 1)
    launch_pdl(ep_dispatch_kernel<1>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.E, El, rank,
               world, PC, xv, expert_idx, slot, kept, cnt_all, xe, local_cnt, status);
  else
    launch_pdl(ep_dispatch_kernel<2>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.E, El, rank,
               world, PC, xv, expert_idx, slot, kept, cnt_all, xe, local_cnt, status);
  const int32_t rc = check_launch("ep_dispatch_kernel");
  if (rc != MOE_OK) return rc;
  launch_pdl(ep_release_kernel, dim3(1), dim3(32), 0, s);
  return check_launch("ep_release_kernel");
}

int32_t launch_ep_combine(const moe_config& c, int rank, int world, const void* const* ye_peers,
                          const int32_t* expert_idx, const float* gate, const int32_t* slot,
                          const uint8_t* kept, const int32_t* cnt_all, void* y, int32_t* status,
                          cudaStream_t s) {
  if (c.T == 0) return MOE_OK;
  const int row_vec = static_cast<int>(c.d_model * elem_size(c.dtype) / 16);
  const int El = c.E / world;
  const int PC = world * c.capacity;
  PeerRowsConst ye{};
  for (int q = 0; q < world && ye_peers; ++q) ye.p[q] = static_cast<const uint4*>(ye_peers[q]);
  const unsigned grid = grid_for_tokens(c.T);
  uint4* yv = static_cast<uint4*>(y);
  if (c.dtype == MOE_DTYPE_BF16) {
    if (c.k == 1)
      launch_pdl(ep_combine_kernel<1, Bf16x8>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.E, El,
                 rank, PC, ye, expert_idx, gate, slot, kept, cnt_all, yv, status);
    else
      launch_pdl(ep_combine_kernel<2, Bf16x8>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.E, El,
                 rank, PC, ye, expert_idx, gate, slot, kept, cnt_all, yv, status);
  } else {
    if (c.k == 1)
      launch_pdl(ep_combine_kernel<1, F32x4>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.E, El,
                 rank, PC, ye, expert_idx, gate, slot, kept, cnt_all, yv, status);
    else
      launch_pdl(ep_combine_kernel<2, F32x4>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.E, El,
                 rank, PC, ye, expert_idx, gate, slot, kept, cnt_all, yv, status);
  }
  return check_launch("ep_combine_kernel");
}

}  // namespace moe
