// Router + softmax gate + top-k on SM pairs (tcgen05 cta_group::2).
//
//   h[t, e] = sum_k x[t, k] Wr[e, k] + bias[e]      (Switch notes sec. 2.1)
//   p[t, e] = exp(h[t, e]) / sum_j exp(h[t, j])     (eq. 1, in fp32: sec. 2.4)
//   expert_idx[t, :k], gate[t, :k] = the k largest p[t, :], ties to the lower e
//
// without writing the logits.  The operation is a skinny GEMM (N = E <= 256)
// whose cost is reading x once, so the design is about the read stream:
//
// * A cluster of two CTAs (one per SM) multiplies 2R tokens by all E rows of
//   W_r with M = 256 MMAs: CTA r holds R <= 128 token rows of the A tile and
//   half of W_r's rows (the B operand's N half), so every SM re-reads only
//   half of W_r per tile.  Rows R..127 of the A stage are never loaded and
//   their accumulator rows are ignored.
// * R is chosen on the host so that the tiles spread evenly over all pairs in
//   whole waves (R = T / (2 * pairs * waves), rounded up to 8 rows): every SM
//   streams the same share of x instead of a few SMs taking one tile more.
// * Each CTA has two TMEM accumulators, so one tile's gate and top-k run
//   while the next is loaded and multiplied, and sixteen epilogue warps, four
//   per TMEM lane quarter: warp set h reads columns [h BN/4, (h+1) BN/4) of
//   its 32 tokens, and sets 1-3 hand their partial results to set 0 through
//   shared memory (a pair of mbarriers per accumulator, bounded waits).
// * Each warp reads its logits from TMEM once (chunks of 32 columns, 16 when
//   E <= 64) and keeps a running maximum, the softmax denominator rescaled at
//   each new maximum, and the running top-1 / top-2 with their indices;
//   inside a chunk the maximum, second and their lowest columns come from
//   pairwise trees.  Chunks and the four quarters are combined in increasing
//   e, and a later part replaces a kept entry only when strictly larger, which
//   gives the (value desc, index asc) order of the top-k definition.
//
// Roles: warp 0 lane 0 of each CTA loads its halves with TMA (both CTAs'
// copies complete on CTA 0's "full" barrier); warp 1 lane 0 of CTA 0 issues
// the MMAs and commits them to both CTAs' barriers; warps 2-17 drain TMEM.
// Every wait is bounded and shares the call's give-up signal; a cluster
// barrier brackets the kernel so neither CTA frees TMEM or exits while its
// partner may still use it.  TMA loads fill only the issuing CTA's own
// shared memory (no multicast).
#include <cuda.h>

#include <algorithm>
#include <climits>
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kHalf = 128;                      // A rows of shared memory per CTA
constexpr int kBK = 64, kUmmaK = 16;
constexpr int kSets = 4;                        // epilogue warp sets (column quarters)
constexpr int kEpiWarps = 4 * kSets;            // one warp of each set per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;   // 576
constexpr int kABytes = kHalf * kBK * 2;        // 16 KB

template <int BN>
struct RCfg {
  static constexpr int kBRows = BN / 2;  // W_r rows per CTA
  static constexpr int kBBytes = kBRows * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (200 * 1024) / kStageBytes > 8 ? 8 : (200 * 1024) / kStageBytes;
  static constexpr int kTmemCols = 2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512);
  static constexpr int kAccStride = kTmemCols / 2;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes;
  static constexpr int kNC = BN / kSets >= 32 ? 32 : 16;  // logits per TMEM load and chunk
  static_assert(BN == 64 || BN == 128 || BN == 256, "N of the pair MMA");
  static_assert(kBBytes % 1024 == 0, "B stage alignment");
};

struct RouterParams {
  int32_t T, E, K;
  int32_t R;       // token rows per CTA and tile (multiple of 8, <= 128)
  int32_t tiles;   // ceil(T / 2R)
  int32_t topk;    // 1 or 2
  const float* bias;     // [E] or null
  int32_t* expert_idx;   // [T, k]
  float* gate;           // [T, k]
  int32_t* status;       // nullable; also the call's give-up signal
  uint64_t wait_ns;
};

// The running result of one token over the logits seen so far.
struct TopState {
  float m;     // maximum (= the top-1 value)
  float s;     // sum of exp(h - m)
  int i1;      // index of the maximum
  float v2;    // second value (top-2)
  int i2;
};

template <int NC>
MOE_DEV float tree_max(float (&w)[NC]) {
#pragma unroll
  for (int n = NC / 2; n > 0; n >>= 1)
#pragma unroll
    for (int i = 0; i < n; ++i) w[i] = fmaxf(w[i], w[i + n]);
  return w[0];
}
template <int NC>
MOE_DEV int tree_min(int (&w)[NC]) {
#pragma unroll
  for (int n = NC / 2; n > 0; n >>= 1)
#pragma unroll
    for (int i = 0; i < n; ++i) w[i] = min(w[i], w[i + n]);
  return w[0];
}

// Merge a part b whose columns all lie above those of the running state a.
template <bool TWO>
MOE_DEV void merge_above(TopState& a, float bm, float bs, int bi1, float bv2, int bi2) {
  // softmax denominators to the common maximum (a part with no finite
  // logit has s = 0 and adds nothing)
  const float m = fmaxf(a.m, bm);
  const float sa = a.s > 0.f ? a.s * __expf(a.m - m) : 0.f;
  const float sb = bs > 0.f ? bs * __expf(bm - m) : 0.f;
  a.s = sa + sb;
  if (bm > a.m) {
    if (TWO) {
      // new second: a's maximum or b's second (tie: a's, the lower index)
      if (a.m >= bv2) { a.v2 = a.m; a.i2 = a.i1; }
      else { a.v2 = bv2; a.i2 = bi2; }
    }
    a.m = bm;
    a.i1 = bi1;
  } else if (TWO && bm > a.v2) {
    a.v2 = bm;
    a.i2 = bi1;
  }
}

// Fold chunk v (columns e0 .. e0 + NC - 1, all above the columns already
// folded) into the running state.
template <bool TWO, int NC>
MOE_DEV void fold_chunk(TopState& st, const float (&v)[NC], int e0) {
  float w[NC];
  int id[NC];
#pragma unroll
  for (int i = 0; i < NC; ++i) w[i] = v[i];
  const float cm = tree_max<NC>(w);
#pragma unroll
  for (int i = 0; i < NC; ++i) id[i] = v[i] == cm ? i : NC;
  const int ci1 = tree_min<NC>(id);
  float cv2 = -INFINITY;
  int ci2 = NC;
  if (TWO) {
#pragma unroll
    for (int i = 0; i < NC; ++i) w[i] = i == ci1 ? -INFINITY : v[i];
    cv2 = tree_max<NC>(w);
#pragma unroll
    for (int i = 0; i < NC; ++i) id[i] = (i != ci1 && v[i] == cv2) ? i : NC;
    ci2 = tree_min<NC>(id);
  }
  float cs = 0.f;
  if (cm > -INFINITY) {
    float part[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) part[i] = 0.f;
#pragma unroll
    for (int i = 0; i < NC; ++i) part[i & 7] += __expf(v[i] - cm);
    cs = ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
  }
  merge_above<TWO>(st, cm, cs, e0 + ci1, cv2, e0 + ci2);
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
router_topk_pair_kernel(const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmW, RouterParams p) {
  using C = RCfg<BN>;
  constexpr int S = C::kStages;
  constexpr uint32_t kIdesc = dev::idesc_bf16_f32(2 * kHalf, BN);

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[S], empty_bar[S], tfull_bar[2], tempty_bar[2], done_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;
  __shared__ float s_bias[BN];
  __shared__ uint64_t part_full[2], part_empty[2];  // set 1 -> set 0 handoff, per accumulator
  __shared__ TopState s_part[2][kSets - 1][kHalf];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* smA = smem;
  uint8_t* smB = smem + S * kABytes;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = dev::cta_rank();
  const int cluster = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;
  const int num_kb = p.K / kBK;
  const int R = p.R;

  dev::pdl_trigger();
  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < S; ++s) {
      dev::mbar_init(&full_bar[s], 1);
      dev::mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      dev::mbar_init(&tfull_bar[a], 1);
      dev::mbar_init(&tempty_bar[a], 2 * kEpiWarps);  // one arrival per epilogue warp, both CTAs
      dev::mbar_init(&part_full[a], (kSets - 1) * 4 * 32);  // sets 1..3's threads
      dev::mbar_init(&part_empty[a], 4 * 32);               // set 0's threads
    }
    dev::mbar_init(&done_bar, 1);
    dev::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    dev::tma_prefetch_desc(&tmX);
    dev::tma_prefetch_desc(&tmW);
  }
  dev::pdl_wait();  // x, W_r and bias may come from the previous kernel
  if (warp == 1) {  // TMEM only after the previous kernel has finished (see pdl_wait)
    dev::tmem_alloc2(&s_tmem_base, C::kTmemCols);
    dev::tmem_relinquish2();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::cluster_sync();  // both CTAs' barriers are initialised and TMEM allocated
  dev::tc_fence_after();
  const uint32_t tmem_base = s_tmem_base;
  const dev::Abort ab{&s_abort, p.status, p.wait_ns};

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      const uint32_t tx = 2u * static_cast<uint32_t>((R + C::kBRows) * kBK * 2);
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      for (int t = cluster; t < p.tiles && !ab.raised_here(); t += n_clusters) {
        const int a_row = t * 2 * R + static_cast<int>(rank) * R;
        const int b_row = static_cast<int>(rank) * C::kBRows;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!dev::mbar_wait(&empty_bar[stage], phase ^ 1u, ab)) break;
          if (rank == 0) dev::mbar_arrive_expect_tx(&full_bar[stage], tx);
          const uint32_t full0 = dev::mapa(&full_bar[stage], 0);
          dev::tma_load_2d_pair(smA + stage * kABytes, &tmX, full0, kb * kBK, a_row);
          dev::tma_load_2d_pair(smB + stage * C::kBBytes, &tmW, full0, kb * kBK, b_row);
          ++issued;
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
      }
      if (rank == 0) {
        // the pair's copies have all landed once CTA 0's full barriers complete
        const unsigned long long deadline = dev::globaltimer() + p.wait_ns;
        for (int s = 0; s < S; ++s) {
          if (issued > s) {
            const long long last_fill = (issued - 1 - s) / S;
            dev::mbar_wait_drain(&full_bar[s], static_cast<uint32_t>(last_fill & 1), ab, deadline);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (CTA 0 only) ----------------
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      for (int t = cluster; t < p.tiles && !ab.raised_here(); t += n_clusters) {
        if (!dev::mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, ab)) break;
        dev::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::kAccStride);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!dev::mbar_wait(&full_bar[stage], phase, ab)) { ok = false; break; }
          dev::tc_fence_after();
          const uint64_t adesc = dev::smem_desc_k_sw128(dev::smem_u32(smA + stage * kABytes));
          const uint64_t bdesc = dev::smem_desc_k_sw128(dev::smem_u32(smB + stage * C::kBBytes));
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk)
            dev::umma2_bf16(d_tmem, adesc + 2ull * kk, bdesc + 2ull * kk, kIdesc,
                            (kb > 0 || kk > 0) ? 1u : 0u);
          dev::umma2_commit_both(&empty_bar[stage]);
          any = true;
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        dev::umma2_commit_both(&tfull_bar[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (any) {
        dev::umma2_commit_local(&done_bar);
        dev::mbar_wait_drain(&done_bar, 0, ab, dev::globaltimer() + p.wait_ns);
      }
    }
  } else {
    // ---------------- epilogue: warps 2..17 ----------------
    const int q = warp & 3;          // TMEM lane quarter this warp may read
    const int h = (warp - 2) >> 2;   // column quarter: [h BN/4, (h+1) BN/4)
    const int row_local = q * 32 + lane;
    // the bias, off the producer's path (named barrier 1: the 256 epilogue threads)
    for (int i = tid - 64; i < BN; i += kThreads - 64)
      s_bias[i] = (p.bias && i < p.E) ? p.bias[i] : 0.f;
    asm volatile("bar.sync 1, %0;" ::"n"(kThreads - 64) : "memory");
    constexpr int NC = C::kNC;
    const int c_lo = h * (BN / kSets);
    const int c_hi = min(c_lo + BN / kSets, p.E);
    const uint32_t tempty0 = dev::mapa(&tempty_bar[0], 0), tempty1 = dev::mapa(&tempty_bar[1], 0);
    const bool two = p.topk == 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = cluster; t < p.tiles; t += n_clusters) {
      int ok = 0;
      if (lane == 0) ok = dev::mbar_wait(&tfull_bar[acc], acc_phase, ab) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      dev::tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * C::kAccStride);
      TopState st{-INFINITY, 0.f, INT_MAX, -INFINITY, INT_MAX};
#pragma unroll 1
      for (int e0 = c_lo; e0 < c_hi; e0 += NC) {
        uint32_t r[NC];
        if constexpr (NC == 32) dev::tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>(e0), r);
        else dev::tmem_ld_32x32b_x16(tbase + static_cast<uint32_t>(e0), r);
        dev::tmem_wait_ld();
        float v[NC];
        if (e0 + NC <= c_hi) {
#pragma unroll
          for (int i = 0; i < NC; ++i) v[i] = __uint_as_float(r[i]) + s_bias[e0 + i];
        } else {  // the last, partial chunk: columns past E take no part
#pragma unroll
          for (int i = 0; i < NC; ++i)
            v[i] = e0 + i < c_hi ? __uint_as_float(r[i]) + s_bias[e0 + i] : -INFINITY;
        }
        if (two) fold_chunk<true, NC>(st, v, e0);
        else fold_chunk<false, NC>(st, v, e0);
      }
      // the accumulator is free for the tile after next
      dev::tc_fence_before();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive_cluster(acc ? tempty1 : tempty0);
      // sets 1..3 -> set 0: slot `acc` of the handoff, its (acc_phase)-th use
      if (h > 0) {
        ok = 0;
        if (lane == 0) ok = dev::mbar_wait(&part_empty[acc], acc_phase ^ 1u, ab) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        s_part[acc][h - 1][row_local] = st;
        dev::mbar_arrive(&part_full[acc]);
      } else {
        ok = 0;
        if (lane == 0) ok = dev::mbar_wait(&part_full[acc], acc_phase, ab) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        TopState o[kSets - 1];
#pragma unroll
        for (int j = 0; j < kSets - 1; ++j) o[j] = s_part[acc][j][row_local];
        dev::mbar_arrive(&part_empty[acc]);
#pragma unroll
        for (int j = 0; j < kSets - 1; ++j) {  // quarters in increasing column order
          if (two) merge_above<true>(st, o[j].m, o[j].s, o[j].i1, o[j].v2, o[j].i2);
          else merge_above<false>(st, o[j].m, o[j].s, o[j].i1, o[j].v2, o[j].i2);
        }
        const int tok = t * 2 * R + static_cast<int>(rank) * R + row_local;
        if (row_local < R && tok < p.T) {
          const float inv = 1.0f / st.s;  // gate of the maximum: exp(m - m) / sum
          if (two) {  // scalar stores: the outputs need only 4-byte alignment
            p.expert_idx[2 * tok] = st.i1;
            p.expert_idx[2 * tok + 1] = st.i2;
            p.gate[2 * tok] = inv;
            p.gate[2 * tok + 1] = expf(st.v2 - st.m) * inv;
          } else {
            p.expert_idx[tok] = st.i1;
            p.gate[tok] = inv;
          }
        }
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  dev::tc_fence_before();
  __syncthreads();
  dev::cluster_sync();  // no CTA frees TMEM or exits while its partner's MMAs or copies may run
  if (warp == 1) {
    __syncwarp();
    dev::tc_fence_after();
    dev::tmem_dealloc2(tmem_base, C::kTmemCols);
  }
}


// Resident pairs of one kernel on this device, queried once per (device, kernel).
template <int BN>
int32_t resident_pairs(int* out) {
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
  using C = RCfg<BN>;
  auto kern = router_topk_pair_kernel<BN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
      cudaSuccess)
    return check_launch("cudaFuncSetAttribute(router_topk_pair_kernel)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms() & ~1));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int resident = 0;
  if (cudaOccupancyMaxActiveClusters(&resident, kern, &cfg) != cudaSuccess || resident < 1)
    return check_launch("cudaOccupancyMaxActiveClusters(router_topk_pair_kernel)");
  if (dev < kMaxDev) cache[dev] = resident;
  *out = resident;
  return MOE_OK;
}

template <int BN>
int32_t launch_router_pair(const moe_config& c, const void* x, const void* Wr, RouterParams p,
                           cudaStream_t s) {
  using C = RCfg<BN>;
  int pairs = 0;
  int32_t rc = resident_pairs<BN>(&pairs);
  if (rc != MOE_OK) return rc;
  // whole waves over all pairs, rows per CTA rounded up to the 8-row swizzle atom
  const int64_t T = c.T;
  const int64_t waves = (T + 2LL * kHalf * pairs - 1) / (2LL * kHalf * pairs);
  int64_t R = (T + 2 * pairs * waves - 1) / (2 * pairs * waves);
  R = (R + 7) & ~int64_t(7);
  if (R > kHalf) R = kHalf;
  p.R = static_cast<int32_t>(R);
  p.tiles = static_cast<int32_t>((T + 2 * R - 1) / (2 * R));
  CUtensorMap tx, tw;
  rc = make_tmap_bf16(&tx, x, static_cast<uint64_t>(c.T), static_cast<uint64_t>(c.d_model),
                 static_cast<uint32_t>(R));
  if (rc != MOE_OK) return rc;
  rc = make_tmap_bf16(&tw, Wr, static_cast<uint64_t>(c.E), static_cast<uint64_t>(c.d_model),
                 static_cast<uint32_t>(C::kBRows));
  if (rc != MOE_OK) return rc;
  auto kern = router_topk_pair_kernel<BN>;
  // on every launch: a function attribute belongs to the current context, the
  // cached pair count to the device
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
      cudaSuccess)
    return check_launch("cudaFuncSetAttribute(router_topk_pair_kernel)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * std::min<int64_t>(pairs, p.tiles)));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaLaunchKernelEx(&cfg, kern, tx, tw, p);
  return check_launch("router_topk_pair_kernel");
}

}  // namespace

// Router with the gate and top-k in its epilogue: expert_idx/gate [T, k]
// without writing logits.
int32_t launch_router_topk_tc(const moe_config& c, const void* x, const void* Wr,
                              const float* bias, int32_t* expert_idx, float* gate,
                              int32_t* status, cudaStream_t s) {
  if (c.T == 0) return MOE_OK;
  RouterParams p{};
  p.T = static_cast<int32_t>(c.T);
  p.E = c.E;
  p.K = c.d_model;
  p.topk = c.k;
  p.bias = bias;
  p.expert_idx = expert_idx;
  p.gate = gate;
  p.status = status;
  p.wait_ns = wait_limit_ns();
  if (c.E <= 64) return launch_router_pair<64>(c, x, Wr, p, s);
  if (c.E <= 128) return launch_router_pair<128>(c, x, Wr, p, s);
  return launch_router_pair<256>(c, x, Wr, p, s);
}

}  // namespace moe
