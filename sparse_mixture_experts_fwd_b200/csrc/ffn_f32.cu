// Expert FFN for fp32 activations (Switch notes sec. 2.1, E_i):
//   H = ReLU(xe W1^T), ye = H W2^T over each expert's kept rows.
// fp32 layers are small (the fp32 workload is a 64-wide, 8-expert layer), so
// this is a plain shared-memory-tiled FMA GEMM grouped over experts: a 16x16
// thread block owns a 16x16 output tile of one expert and skips tiles past
// the expert's kept-row count.  bf16 layers use the tensor-core GEMM.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kTile = 16;

template <bool RELU>
__global__ void __launch_bounds__(kTile * kTile) grouped_gemm_f32_kernel(
    int N, int K, int C, const int32_t* __restrict__ rows_per_group, const float* __restrict__ A,
    const float* __restrict__ B, float* __restrict__ out) {
  dev::pdl_trigger();
  dev::pdl_wait();
  const int g = blockIdx.z;
  int rows = __ldg(rows_per_group + g);
  rows = rows < 0 ? 0 : (rows > C ? C : rows);
  const int m0 = blockIdx.y * kTile;
  if (m0 >= rows) return;
  const int n0 = blockIdx.x * kTile;
  __shared__ float sA[kTile][kTile + 1], sB[kTile][kTile + 1];
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int64_t a_base = static_cast<int64_t>(g) * C;
  const int64_t b_base = static_cast<int64_t>(g) * N;
  float acc = 0.f;
  for (int k0 = 0; k0 < K; k0 += kTile) {
    const int kk = k0 + tx;
    const int m = m0 + ty;
    const int n = n0 + ty;
    sA[ty][tx] = (m < rows && kk < K) ? __ldg(A + (a_base + m) * K + kk) : 0.f;
    sB[ty][tx] = (n < N && kk < K) ? __ldg(B + (b_base + n) * K + kk) : 0.f;
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kTile; ++q) acc = fmaf(sA[ty][q], sB[tx][q], acc);
    __syncthreads();
  }
  const int m = m0 + ty, n = n0 + tx;
  if (m < rows && n < N) out[(a_base + m) * N + n] = RELU ? fmaxf(acc, 0.f) : acc;
}

}  // namespace

int32_t launch_ffn_f32(const moe_config& c, const void* xe, const void* W1, const void* W2,
                       const int32_t* kept_cnt, void* H, void* ye, cudaStream_t s) {
  if (c.E == 0 || c.capacity == 0) return MOE_OK;
  const dim3 block(kTile, kTile);
  const unsigned my = static_cast<unsigned>((c.capacity + kTile - 1) / kTile);
  dim3 g1((c.d_ff + kTile - 1) / kTile, my, c.E);
  launch_pdl(grouped_gemm_f32_kernel<true>, dim3(g1), dim3(block), 0, s, c.d_ff, c.d_model, c.capacity, kept_cnt,
                                                     static_cast<const float*>(xe),
                                                     static_cast<const float*>(W1),
                                                     static_cast<float*>(H));
  int32_t rc = check_launch("grouped_gemm_f32_kernel (W1)");
  if (rc != MOE_OK) return rc;
  dim3 g2((c.d_model + kTile - 1) / kTile, my, c.E);
  launch_pdl(grouped_gemm_f32_kernel<false>, dim3(g2), dim3(block), 0, s, c.d_model, c.d_ff, c.capacity, kept_cnt,
                                                      static_cast<const float*>(H),
                                                      static_cast<const float*>(W2),
                                                      static_cast<float*>(ye));
  return check_launch("grouped_gemm_f32_kernel (W2)");
}

}  // namespace moe
