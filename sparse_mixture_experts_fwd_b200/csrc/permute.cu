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
#include <algorithm>

#include "moe_internal.cuh"

namespace moe {
namespace {

template <int K>
__global__ void __launch_bounds__(256) dispatch_kernel(int64_t T, int row_vec, int C,
                                                       const uint4* __restrict__ x,
                                                       const int32_t* __restrict__ expert_idx,
                                                       const int32_t* __restrict__ slot,
                                                       const uint8_t* __restrict__ kept,
                                                       uint4* __restrict__ xe,
                                                       unsigned int* __restrict__ zero_words,
                                                       int n_zero, uint4* __restrict__ y_zero) {
  dev::pdl_trigger();
  dev::pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  // counters the next kernel on this stream expects at zero (the fused expert FFN)
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero_words[i] = 0u;
  for (int64_t t = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5; t < T;
       t += nwarps) {
    int64_t dst[K];
    int nd = 0;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      if (__ldg(kept + t * K + j)) {
        dst[nd++] = (static_cast<int64_t>(__ldg(expert_idx + t * K + j)) * C +
                     __ldg(slot + t * K + j)) * row_vec;
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
      xe[dst[0] + v] = val;
      if (K == 2 && nd == 2) xe[dst[K - 1] + v] = val;
    }
  }
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
__global__ void __launch_bounds__(256) combine_kernel(int64_t T, int row_vec, int C,
                                                      const uint4* __restrict__ ye,
                                                      const int32_t* __restrict__ expert_idx,
                                                      const float* __restrict__ gate,
                                                      const int32_t* __restrict__ slot,
                                                      const uint8_t* __restrict__ kept,
                                                      uint4* __restrict__ y) {
  dev::pdl_trigger();
  dev::pdl_wait();
  constexpr int N = V::kN;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t t = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5; t < T;
       t += nwarps) {
    int64_t src[K];
    float g[K];
    int ns = 0;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      if (__ldg(kept + t * K + j)) {
        src[ns] = (static_cast<int64_t>(__ldg(expert_idx + t * K + j)) * C +
                   __ldg(slot + t * K + j)) * row_vec;
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
}

unsigned grid_for_tokens(int64_t T) {
  const int64_t want = (T + 7) / 8;  // 8 warps per block, a warp per token
  return static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(want, int64_t(num_sms()) * 16)));
}

}  // namespace

int32_t launch_dispatch(const moe_config& c, const void* x, const int32_t* expert_idx,
                        const int32_t* slot, const uint8_t* kept, void* xe, cudaStream_t s,
                        unsigned int* zero_words, int n_zero, void* y_zero) {
  if (c.T == 0 || (c.capacity == 0 && !y_zero)) return MOE_OK;
  const int row_vec = static_cast<int>(c.d_model * elem_size(c.dtype) / 16);
  const unsigned grid = grid_for_tokens(c.T);
  uint4* yz = static_cast<uint4*>(y_zero);
  if (c.k == 1)
    launch_pdl(dispatch_kernel<1>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.capacity,
               static_cast<const uint4*>(x), expert_idx, slot, kept, static_cast<uint4*>(xe),
               zero_words, n_zero, yz);
  else
    launch_pdl(dispatch_kernel<2>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.capacity,
               static_cast<const uint4*>(x), expert_idx, slot, kept, static_cast<uint4*>(xe),
               zero_words, n_zero, yz);
  return check_launch("dispatch_kernel");
}

int32_t launch_combine(const moe_config& c, const void* ye, const int32_t* expert_idx,
                       const float* gate, const int32_t* slot, const uint8_t* kept, void* y,
                       cudaStream_t s) {
  if (c.T == 0) return MOE_OK;
  const int row_vec = static_cast<int>(c.d_model * elem_size(c.dtype) / 16);
  const unsigned grid = grid_for_tokens(c.T);
  const uint4* yev = static_cast<const uint4*>(ye);
  uint4* yv = static_cast<uint4*>(y);
  if (c.dtype == MOE_DTYPE_BF16) {
    if (c.k == 1)
      launch_pdl(combine_kernel<1, Bf16x8>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.capacity, yev, expert_idx,
                                                     gate, slot, kept, yv);
    else
      launch_pdl(combine_kernel<2, Bf16x8>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.capacity, yev, expert_idx,
                                                     gate, slot, kept, yv);
  } else {
    if (c.k == 1)
      launch_pdl(combine_kernel<1, F32x4>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.capacity, yev, expert_idx,
                                                    gate, slot, kept, yv);
    else
      launch_pdl(combine_kernel<2, F32x4>, dim3(grid), dim3(256), 0, s, c.T, row_vec, c.capacity, yev, expert_idx,
                                                    gate, slot, kept, yv);
  }
  return check_launch("combine_kernel");
}

}  // namespace moe
