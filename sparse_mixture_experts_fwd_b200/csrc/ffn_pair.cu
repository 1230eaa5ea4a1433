// Expert FFN for bf16 layers whose experts hold hundreds of rows (Switch
// notes sec. 2.1, the experts E_i; tensor-core bound):
//   H[e]  = round(act(xe[e] W1[e]^T))      GEMM 1, K = d_model
//   out   = round(g * (H[e] W2[e]^T))      GEMM 2, K = d_ff
// as ONE persistent kernel on SM pairs (tcgen05 cta_group::2).
//
// Orientation: the weights are the MMA's M side and the tokens its N side.
// A tile is 256 output features (W1 or W2 rows) x N tokens of one expert,
// N <= 256 in steps of 16: an expert's r kept rows are cut into chunks of 256
// rows and one of the rest, rounded up to 16, so an expert with 530 rows
// computes 544 token columns instead of three 256-row blocks (768).  CTA r
// of the pair holds features [128r, 128r + 128) of the tile (its half of the
// A operand) and tokens [rN/2, rN/2 + N/2) of the chunk (its half of B); its
// TMEM lanes are its 128 features and the columns the N tokens.  The token
// half is fetched as one TMA box of 128, 64, 32, 16 or 8 rows, the smallest
// that holds it (one load per operand and stage: more, smaller boxes per
// stage left the MMAs waiting on the TMA unit).

// Both GEMMs run in one tile sequence of "units" (unit u: the GEMM-1 tiles
// of expert u, then the GEMM-2 tiles of expert u - L), tiles of one expert
// ordered (feature block, chunk) so the chunks sharing a weight tile run side
// by side and read it from L2.  CTA 0 of each pair takes tiles from a global
// counter one tile ahead and publishes each to both CTAs through a
// shared-memory ring in the cluster one tile before its loads begin, so the
// load balances to within one tile, there is no tail between the GEMMs and a
// pair that is not yet running holds no tile.  A GEMM-2 tile of (expert,
// chunk) needs every GEMM-1 tile of that chunk: each epilogue warp that
// stored its part of a GEMM-1 tile adds one (release) to the chunk's counter,
// and the producers of a GEMM-2 tile wait (acquire, bounded) for 16 per
// GEMM-1 feature block.  H of the experts in flight stays in L2.
//
// Epilogue: an accumulator column is one token, a lane one feature, so each
// warp packs a lane's two tokens into a bf16x2 word, swaps it with the
// neighbour lane and stores 4 bytes per lane: every store instruction writes
// two 64-byte runs of two token rows.  GEGLU: lanes 2i, 2i + 1 hold hidden
// unit i's gate and linear parts.  Top-1 layers: GEMM 2 writes gate * row
// straight to y in token order.  Two accumulators in tensor memory let a
// tile's epilogue run under the next tile's MMAs; eight warps (two per lane
// quarter, alternate 32-column blocks) keep it shorter than a short-K tile's
// main loop.

// Roles per CTA (320 threads): warp 0 lane 0 loads this CTA's halves (CTA 0's
// also takes tiles); warp 1 lane 0 of CTA 0 issues the MMAs (M = 256) and
// commits them to both CTAs; warps 2-9 drain their CTA's TMEM.  Every wait is
// bounded and shares the call's give-up signal; TMA loads fill only the
// issuing CTA's shared memory (no multicast).
#include <cuda.h>

#include <algorithm>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kHalf = 128;                 // A rows (features) per CTA
constexpr int kBM = 256;                   // features per tile
constexpr int kMaxN = 256;                 // tokens per tile (one accumulator)
constexpr int kChunk = kMaxN;              // rows per chunk of an expert
constexpr int kBK = 64, kUmmaK = 16;
constexpr int kEpiWarps = 8;               // two per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kStages = 6;
constexpr int kRing = 8;
constexpr int kABytes = kHalf * kBK * 2;          // 16 KB
constexpr int kBRowsMax = kMaxN / 2;              // token rows per CTA
constexpr int kBBytesMax = kBRowsMax * kBK * 2;   // 16 KB
constexpr int kStageBytes = kABytes + kBBytesMax;
constexpr int kTmemCols = 512;
constexpr int kMaxE = 256;
constexpr int kMaxUnits = 2 * kMaxE;
constexpr int kSmemBytes = 1024 + kStages * kStageBytes;
constexpr int kBoxes = 5;                 // token-row boxes of 128, 64, 32, 16, 8 rows
constexpr int kCtrPerTile = 2 * kEpiWarps;  // counter arrivals per GEMM-1 tile: both CTAs' warps

struct Maps {
  CUtensorMap w1;           // W1 [E * n1, d], box 128 x 64
  CUtensorMap w2;           // W2 [E * d, f], box 128 x 64
  CUtensorMap x[kBoxes];    // xe [E * C, d], box (128 >> i) x 64
  CUtensorMap h[kBoxes];    // H  [E * C, f], box (128 >> i) x 64
};

struct PairParams {
  int E, C, d, f, n1, lag, maxc;
  int nm1, nm2;             // 256-feature blocks of GEMM 1 (n1 rows) and GEMM 2 (d rows)
  int glu;
  const int32_t* kept_cnt;
  __nv_bfloat16* H;
  __nv_bfloat16* ye;
  unsigned int* tile_ctr;   // zero before launch
  unsigned int* chunk_ctr;  // [E * maxc], zero before launch
  int32_t* status;          // nullable; also the call's give-up signal
  uint64_t wait_ns;
  const int32_t* tok_of_row;  // top-1: row -> token map; null -> write ye
  const float* gate;
  __nv_bfloat16* y;
};

// Shape of the tile of chunk c of an expert with r kept rows: N columns, the
// first N / 2 rows in CTA 0's half of B, the rest in CTA 1's.
struct Geo {
  int row0;   // first row of the chunk within the expert
  int rows;   // rows (tokens) of the chunk
  int N;      // MMA N
  int half;   // token rows per CTA (B operand)
};
MOE_DEV Geo chunk_geo(int r, int c) {
  Geo g;
  g.row0 = c * kChunk;
  g.rows = min(kChunk, r - g.row0);
  g.N = (g.rows + 15) / 16 * 16;
  g.half = g.N / 2;
  return g;
}

struct Tile {
  int kind;  // 1: GEMM 1, 2: GEMM 2
  int e, m, c;
};

// Per-expert chunking and the unit sequence, built in shared memory.
struct Sched {
  int E, lag, nm1, nm2, units;
  const int* nc;      // chunks per expert
  const int* prefix;  // [units + 1]

  __device__ int g1(int u) const { return u < E ? nm1 * nc[u] : 0; }
  __device__ int g2(int u) const { return (u >= lag && u - lag < E) ? nm2 * nc[u - lag] : 0; }

  __device__ Tile decode(int t) const {
    int lo = 0, hi = units - 1;  // last unit with prefix <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
    }
    int local = t - prefix[lo];
    Tile x;
    const int a = g1(lo);
    if (local < a) {
      x.kind = 1;
      x.e = lo;
    } else {
      local -= a;
      x.kind = 2;
      x.e = lo - lag;
    }
    x.m = local / nc[x.e];
    x.c = local - x.m * nc[x.e];
    return x;
  }
};

// ---- cluster helpers (shared ones in moe_internal.cuh) ----
using dev::cluster_sync;
using dev::cta_rank;
using dev::mapa;
using dev::mbar_arrive_cluster;
using dev::mbar_wait_cluster;
using dev::st_cluster_u32;
using dev::tma_load_2d_pair;
using dev::tmem_alloc2;
using dev::tmem_dealloc2;
using dev::tmem_relinquish2;
using dev::umma2_bf16;
using dev::umma2_commit_both;
using dev::umma2_commit_local;

MOE_DEV unsigned int ld_acquire_u32(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
MOE_DEV void red_release_add_u32(unsigned int* p, unsigned int v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
MOE_DEV void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Bounded wait until *p - need >= 0 as a signed difference (acquire).
MOE_DEV bool wait_count(const unsigned int* p, unsigned int need, const dev::Abort& ab) {
  if (static_cast<int>(ld_acquire_u32(p) - need) >= 0) return true;
  const unsigned long long t0 = dev::globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (static_cast<int>(ld_acquire_u32(p) - need) >= 0) return true;
    if ((it & 15u) == 0) {
      if (ab.raised()) return false;
      if (dev::globaltimer() - t0 > ab.limit_ns) {
        ab.raise();
        return false;
      }
      __nanosleep(64);
    }
  }
}


// bf16x2 of (lo, hi) rounded to nearest even, lo in the low half; RELU also
// clamps each to >= 0 (cvt's .relu: the rounding keeps the sign, so it is the
// same as clamping first)
template <bool RELU>
MOE_DEV uint32_t cvt_pair(float lo, float hi) {
  uint32_t d;
  if (RELU)
    asm("cvt.rn.relu.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  else
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// Stores one 32-lane x NC-column accumulator block of a ReLU / plain tile:
// lane = feature fe0 + lane, column n0 + j = chunk row n0 + j.  Each lane
// packs its feature at rows (2j, 2j + 1) into one bf16x2 word and trades it
// with its neighbour lane, so lane 2i stores features (2i, 2i + 1) of row 2j
// and lane 2i + 1 those of row 2j + 1, 4 bytes each.
template <int NC, bool RELU, bool SCATTER>
MOE_DEV void store_pairs(const uint32_t (&r)[32], int lane, const Geo& g, int n0,
                         __nv_bfloat16* out, int64_t row_base, int64_t ld, int fe, bool fe_ok,
                         int tok_lane, float g_lane) {
  const int p = lane & 1;
#pragma unroll
  for (int j = 0; j < NC / 2; ++j) {
    float v0 = __uint_as_float(r[2 * j]), v1 = __uint_as_float(r[2 * j + 1]);
    int tok = 0;
    if (SCATTER) {
      v0 *= __shfl_sync(0xffffffffu, g_lane, 2 * j);
      v1 *= __shfl_sync(0xffffffffu, g_lane, 2 * j + 1);
      tok = __shfl_sync(0xffffffffu, tok_lane, 2 * j + p);
    }
    const uint32_t mine = cvt_pair<RELU>(v0, v1);          // my feature, columns 2j | 2j+1
    const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
    // even lane: (mine.lo, other.lo) = column 2j; odd lane: (other.hi, mine.hi) = column 2j+1
    const uint32_t w = p ? __byte_perm(other, mine, 0x7632) : __byte_perm(mine, other, 0x5410);
    const int row = n0 + 2 * j + p;
    if (fe_ok && row < g.rows) {
      const int64_t orow = SCATTER ? static_cast<int64_t>(tok) : row_base + row;
      *reinterpret_cast<uint32_t*>(out + orow * ld + fe) = w;
    }
  }
}

// GEGLU GEMM-1 block: lanes 4k, 4k + 1 hold hidden unit 2k's gate and linear
// rows, lanes 4k + 2, 4k + 3 unit 2k + 1's.  Even lanes form GELU(g) * l of
// the even columns, odd lanes of the odd ones; then lanes L and L ^ 2 trade
// values so that each stores units (2k, 2k + 1) of one row in 4 bytes.
template <int NC>
MOE_DEV void store_geglu(const uint32_t (&r)[32], int lane, const Geo& g, int n0,
                         __nv_bfloat16* out, int64_t row_base, int64_t ld, int unit_even,
                         bool unit_ok) {
  const int p = lane & 1;        // column parity this lane finishes
  const int s = (lane >> 1) & 1; // 0: unit 2k, 1: unit 2k + 1
  float h[NC / 2];
#pragma unroll
  for (int j = 0; j < NC / 2; ++j) {
    // lane 2i (gate) needs the linear part of column 2j, lane 2i + 1 the gate of column 2j + 1
    const float mine0 = __uint_as_float(r[2 * j]), mine1 = __uint_as_float(r[2 * j + 1]);
    const float other = __shfl_xor_sync(0xffffffffu, p ? mine0 : mine1, 1);
    const float gt = p ? other : mine0;
    const float l = p ? mine1 : other;
    h[j] = dev::geglu(gt, l);  // unit u(lane) at column 2j + p
  }
#pragma unroll
  for (int i = 0; i < NC / 4; ++i) {
    const float send = s ? h[2 * i] : h[2 * i + 1];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 2);
    const uint32_t w = cvt_pair<false>(s ? recv : h[2 * i],       // unit 2k
                                       s ? h[2 * i + 1] : recv);  // unit 2k + 1
    const int row = n0 + 4 * i + 2 * s + p;
    if (unit_ok && row < g.rows)
      *reinterpret_cast<uint32_t*>(out + (row_base + row) * ld + unit_even) = w;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
ffn_pair_kernel(const __grid_constant__ Maps maps, PairParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[kStages], empty_bar[kStages], tfull_bar[2], tempty_bar[2], done_bar;
  __shared__ uint64_t ring_full[kRing], ring_empty[kRing];
  __shared__ int s_ring[kRing];
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_rows[kMaxE], s_nc[kMaxE], s_prefix[kMaxUnits + 1];
  __shared__ volatile int s_abort;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* smA = smem;
  uint8_t* smB = smem + kStages * kABytes;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cta_rank();
  const int E = p.E;
  Sched sc;
  sc.E = E;
  sc.lag = p.lag;
  sc.nm1 = p.nm1;
  sc.nm2 = p.nm2;
  sc.units = E + p.lag;
  sc.nc = s_nc;
  sc.prefix = s_prefix;

  dev::pdl_trigger();
  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < kStages; ++s) {
      dev::mbar_init(&full_bar[s], 1);
      dev::mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      dev::mbar_init(&tfull_bar[a], 1);
      dev::mbar_init(&tempty_bar[a], 2 * 32 * kEpiWarps);  // epilogue threads of both CTAs (CTA 0's used)
    }
    for (int r = 0; r < kRing; ++r) {
      dev::mbar_init(&ring_full[r], 1);
      // CTA 0's: its MMA lane and epilogue warps, CTA 1's producer and epilogue warps
      dev::mbar_init(&ring_empty[r], 2 + 2 * kEpiWarps);
    }
    dev::mbar_init(&done_bar, 1);
    dev::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    dev::tma_prefetch_desc(&maps.w1);
    dev::tma_prefetch_desc(&maps.w2);
  }
  dev::pdl_wait();  // kept counts, xe and the zeroed counters are visible from here
  if (warp == 1) {  // TMEM only after the previous kernel has finished (see pdl_wait)
    tmem_alloc2(&s_tmem_base, kTmemCols);
    tmem_relinquish2();
  }
  for (int e = tid; e < E; e += kThreads) {
    int r = p.kept_cnt[e];
    r = r < 0 ? 0 : (r > p.C ? p.C : r);
    s_rows[e] = r;
    s_nc[e] = (r + kChunk - 1) / kChunk;  // chunks of 256 rows, the last one the rest
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int u = 0; u < sc.units; ++u) {
      s_prefix[u] = acc;
      acc += sc.g1(u) + sc.g2(u);
    }
    s_prefix[sc.units] = acc;
  }
  dev::tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised and TMEM allocated
  dev::tc_fence_after();
  const uint32_t tmem_base = s_tmem_base;
  const int total = s_prefix[sc.units];
  const dev::Abort ab{&s_abort, p.status, p.wait_ns};
  const uint32_t ring_empty0 = mapa(&ring_empty[0], 0);  // CTA 0's ring_empty[0]
  const uint32_t ring_stride = static_cast<uint32_t>(sizeof(uint64_t));

  if (warp == 0) {
    // ---------------- tile taker (CTA 0) + TMA producer (both CTAs) ----------------
    if (lane == 0) {
      int slot = 0;            // CTA 1: next ring slot to read
      uint32_t rphase = 0;
      int pslot = 0;           // CTA 0: next ring slot to write
      uint32_t pphase = 0;
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      // CTA 0 publishes each tile one tile before it loads it, and takes it
      // from the counter one tile before that: CTA 1 starts its loads of a
      // tile as early as CTA 0, and no atomic round trip sits between tiles
      auto clamp_tile = [&](unsigned int v) {
        const int t = static_cast<int>(v);
        return (t < 0 || t >= total) ? -1 : t;  // (negative only from a counter not zeroed)
      };
      auto publish = [&](int t) -> bool {
        if (!mbar_wait_cluster(&ring_empty[pslot], pphase ^ 1u, ab)) return false;
        s_ring[pslot] = t;
        st_cluster_u32(mapa(&s_ring[pslot], 1), t);
        dev::mbar_arrive(&ring_full[pslot]);
        mbar_arrive_cluster(mapa(&ring_full[pslot], 1));
        if (++pslot == kRing) { pslot = 0; pphase ^= 1u; }
        return true;
      };
      int cur = -1;
      unsigned int pending = 0u;
      bool run = true;
      if (rank == 0) {
        cur = clamp_tile(atomicAdd(p.tile_ctr, 1u));
        run = publish(cur);
        if (cur >= 0) pending = atomicAdd(p.tile_ctr, 1u);
      }
      while (run && !ab.raised_here()) {
        int t;
        if (rank == 0) {
          t = cur;
          if (t < 0) break;
          const int nxt = clamp_tile(pending);  // taken one tile ago
          if (!publish(nxt)) break;
          if (nxt >= 0) pending = atomicAdd(p.tile_ctr, 1u);
          cur = nxt;
        } else {
          if (!mbar_wait_cluster(&ring_full[slot], rphase, ab)) break;
          t = s_ring[slot];
          mbar_arrive_cluster(ring_empty0 + static_cast<uint32_t>(slot) * ring_stride);
          if (++slot == kRing) { slot = 0; rphase ^= 1u; }
        }
        if (t < 0) break;
        const Tile x = sc.decode(t);
        const Geo g = chunk_geo(s_rows[x.e], x.c);
        const CUtensorMap* ta = x.kind == 1 ? &maps.w1 : &maps.w2;
        const CUtensorMap* tb = x.kind == 1 ? maps.x : maps.h;
        const int K = x.kind == 1 ? p.d : p.f;
        const int a_row = x.e * (x.kind == 1 ? p.n1 : p.d) + x.m * kBM + static_cast<int>(rank) * kHalf;
        const int b_row = x.e * p.C + g.row0 + static_cast<int>(rank) * g.half;
        if (x.kind == 2) {
          // every GEMM-1 tile of this chunk must have stored its slice of H
          const unsigned int need = static_cast<unsigned int>(kCtrPerTile * p.nm1);
          if (!wait_count(p.chunk_ctr + x.e * p.maxc + x.c, need, ab)) break;
          fence_proxy_async_global();  // generic-proxy H stores -> async-proxy (TMA) reads
        }
        // the CTA's token rows are one box of the smallest of 256/128/.../8
        // rows that holds them: one TMA per operand and stage (rows past the
        // chunk load but no MMA reads them)
        int box = 0;
        while (box + 1 < kBoxes && (kBRowsMax >> (box + 1)) >= g.half) ++box;
        const uint32_t tx = static_cast<uint32_t>(2 * (kABytes + (kBRowsMax >> box) * kBK * 2));
        bool ok = true;
        for (int kb = 0; kb < K / kBK; ++kb) {
          if (!dev::mbar_wait(&empty_bar[stage], phase ^ 1u, ab)) { ok = false; break; }
          if (rank == 0) dev::mbar_arrive_expect_tx(&full_bar[stage], tx);
          const uint32_t full0 = mapa(&full_bar[stage], 0);
          tma_load_2d_pair(smA + stage * kABytes, ta, full0, kb * kBK, a_row);
          tma_load_2d_pair(smB + stage * kBBytesMax, tb + box, full0, kb * kBK, b_row);
          ++issued;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // no bulk copy may still be landing in shared memory when the CTA exits:
      // CTA 0's full barriers see both CTAs' bytes; CTA 1 waits until the MMAs
      // have released each stage it filled (or the drain deadline)
      const unsigned long long deadline = dev::globaltimer() + p.wait_ns;
      for (int s = 0; s < kStages; ++s) {
        if (issued > s) {
          const long long last_fill = (issued - 1 - s) / kStages;
          if (rank == 0)
            dev::mbar_wait_drain(&full_bar[s], static_cast<uint32_t>(last_fill & 1), ab, deadline);
          else
            dev::mbar_wait_drain(&empty_bar[s], static_cast<uint32_t>(last_fill & 1), ab, deadline);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (CTA 0) ----------------
    if (lane == 0 && rank == 0) {
      int slot = 0;
      uint32_t rphase = 0;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      while (true) {
        if (!mbar_wait_cluster(&ring_full[slot], rphase, ab)) break;
        const int t = s_ring[slot];
        dev::mbar_arrive(&ring_empty[slot]);
        if (++slot == kRing) { slot = 0; rphase ^= 1u; }
        if (t < 0) break;
        const Tile x = sc.decode(t);
        const Geo g = chunk_geo(s_rows[x.e], x.c);
        const uint32_t idesc = dev::idesc_bf16_f32(kBM, g.N);
        const int num_kb = (x.kind == 1 ? p.d : p.f) / kBK;
        if (!dev::mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, ab)) break;
        dev::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kMaxN);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!dev::mbar_wait(&full_bar[stage], phase, ab)) { ok = false; break; }
          dev::tc_fence_after();
          const uint64_t adesc = dev::smem_desc_k_sw128(dev::smem_u32(smA + stage * kABytes));
          const uint64_t bdesc = dev::smem_desc_k_sw128(dev::smem_u32(smB + stage * kBBytesMax));
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk)
            umma2_bf16(d_tmem, adesc + 2ull * kk, bdesc + 2ull * kk, idesc,
                       (kb > 0 || kk > 0) ? 1u : 0u);
          umma2_commit_both(&empty_bar[stage]);
          any = true;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma2_commit_both(&tfull_bar[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (any) {
        umma2_commit_local(&done_bar);
        dev::mbar_wait_drain(&done_bar, 0, ab, dev::globaltimer() + p.wait_ns);
      }
    }
  } else {
    // ---------------- epilogue: warps 2..9 of both CTAs ----------------
    const int q = warp & 3;          // TMEM lane quarter this warp may read
    const int hsel = (warp - 2) >> 2;  // which alternate 32-column blocks it stores
    const uint32_t tempty_c0 = mapa(&tempty_bar[0], 0);
    const uint32_t tempty_c1 = mapa(&tempty_bar[1], 0);
    int slot = 0;
    uint32_t rphase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    while (true) {
      int t = -1, ok = 0;
      if (lane == 0) {
        ok = mbar_wait_cluster(&ring_full[slot], rphase, ab) ? 1 : 0;
        if (ok) {
          t = s_ring[slot];
          if (rank == 0) dev::mbar_arrive(&ring_empty[slot]);
          else mbar_arrive_cluster(ring_empty0 + static_cast<uint32_t>(slot) * ring_stride);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      t = __shfl_sync(0xffffffffu, t, 0);
      if (!ok || t < 0) break;
      if (++slot == kRing) { slot = 0; rphase ^= 1u; }
      const Tile x = sc.decode(t);
      if (lane == 0) ok = dev::mbar_wait(&tfull_bar[acc], acc_phase, ab) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      dev::tc_fence_after();
      const Geo g = chunk_geo(s_rows[x.e], x.c);
      const int feat = x.m * kBM + static_cast<int>(rank) * kHalf + q * 32 + lane;  // this lane's
      const int64_t row_base = static_cast<int64_t>(x.e) * p.C + g.row0;
      for (int n0 = 32 * hsel; n0 < g.N; n0 += 64) {
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>(acc * kMaxN + n0);
        uint32_t r[32];
        const bool full = g.N - n0 >= 32;
        if (full) {
          dev::tmem_ld_32x32b_x32(taddr, r);
        } else {
          uint32_t r16[16];
          dev::tmem_ld_32x32b_x16(taddr, r16);
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = r16[i];
        }
        dev::tmem_wait_ld();
        if (x.kind == 1) {
          if (p.glu) {
            const int unit_even = (feat >> 2) << 1;
            const bool unit_ok = feat < p.n1;
            if (full) store_geglu<32>(r, lane, g, n0, p.H, row_base, p.f, unit_even, unit_ok);
            else store_geglu<16>(r, lane, g, n0, p.H, row_base, p.f, unit_even, unit_ok);
          } else {
            const int fe = feat & ~1;
            const bool fe_ok = fe < p.n1;
            if (full)
              store_pairs<32, true, false>(r, lane, g, n0, p.H, row_base, p.f, fe, fe_ok, 0, 1.f);
            else
              store_pairs<16, true, false>(r, lane, g, n0, p.H, row_base, p.f, fe, fe_ok, 0, 1.f);
          }
        } else {
          const int fe = feat & ~1;
          const bool fe_ok = fe < p.d;
          if (p.y) {
            // top-1 combine: y[t] = gate_t * E(x_t), into token order
            int tok_lane = 0;
            float g_lane = 1.f;
            if (n0 + lane < g.rows) {
              tok_lane = __ldg(p.tok_of_row + row_base + n0 + lane);
              g_lane = __ldg(p.gate + tok_lane);
            }
            if (full)
              store_pairs<32, false, true>(r, lane, g, n0, p.y, 0, p.d, fe, fe_ok, tok_lane, g_lane);
            else
              store_pairs<16, false, true>(r, lane, g, n0, p.y, 0, p.d, fe, fe_ok, tok_lane, g_lane);
          } else {
            if (full)
              store_pairs<32, false, false>(r, lane, g, n0, p.ye, row_base, p.d, fe, fe_ok, 0, 1.f);
            else
              store_pairs<16, false, false>(r, lane, g, n0, p.ye, row_base, p.d, fe, fe_ok, 0, 1.f);
          }
        }
      }
      dev::tc_fence_before();
      mbar_arrive_cluster(acc == 0 ? tempty_c0 : tempty_c1);  // CTA 0's accumulator-free barrier
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      if (x.kind == 1) {
        // publish this warp's part of H for the chunk: its stores are fenced,
        // then one release increment per warp
        fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) red_release_add_u32(p.chunk_ctr + x.e * p.maxc + x.c, 1u);
      }
    }
  }

  dev::tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA frees TMEM or exits while its partner's MMAs or copies may run
  if (warp == 1) {
    __syncwarp();
    dev::tc_fence_after();
    tmem_dealloc2(tmem_base, kTmemCols);
  }
}

}  // namespace

int ffn_pair_chunks(const moe_config& c) {
  return std::max(1, (c.capacity + kChunk - 1) / kChunk);
}

int32_t launch_ffn_pair_fused(const moe_config& c, const void* xe, const void* W1, const void* W2,
                              const int32_t* kept_cnt, void* H, void* ye, void* sync,
                              bool sync_zeroed, int32_t* status, cudaStream_t s,
                              const Top1Out* top1) {
  const int64_t E = c.E, C = c.capacity, d = c.d_model, f = c.d_ff;
  if (E == 0 || C == 0) return MOE_OK;
  if (E > kMaxE) return fail(MOE_ERR_UNSUPPORTED, "ffn_pair_kernel: E > 256");
  const int maxc = ffn_pair_chunks(c);
  if (!sync_zeroed) {
    cudaError_t e = cudaMemsetAsync(sync, 0, ffn_sync_bytes(c), s);
    if (e != cudaSuccess)
      return fail(MOE_ERR_CUDA, std::string("cudaMemsetAsync: ") + cudaGetErrorString(e));
  }
  const bool glu = c.expert == MOE_EXPERT_GEGLU;
  const int64_t n1 = glu ? 2 * f : f;  // W1 rows per expert
  Maps maps;
  int32_t rc = make_tmap_bf16(&maps.w1, W1, static_cast<uint64_t>(E * n1), static_cast<uint64_t>(d), kHalf);
  if (rc == MOE_OK) rc = make_tmap_bf16(&maps.w2, W2, static_cast<uint64_t>(E * d), static_cast<uint64_t>(f), kHalf);
  for (int i = 0; i < kBoxes && rc == MOE_OK; ++i) {
    rc = make_tmap_bf16(&maps.x[i], xe, static_cast<uint64_t>(E * C), static_cast<uint64_t>(d),
                   kBRowsMax >> i);
    if (rc == MOE_OK)
      rc = make_tmap_bf16(&maps.h[i], H, static_cast<uint64_t>(E * C), static_cast<uint64_t>(f),
                     kBRowsMax >> i);
  }
  if (rc != MOE_OK) return rc;
  PairParams p{};
  p.E = c.E;
  p.C = c.capacity;
  p.d = c.d_model;
  p.f = c.d_ff;
  p.n1 = static_cast<int>(n1);
  p.maxc = maxc;
  p.nm1 = static_cast<int>((n1 + kBM - 1) / kBM);
  p.nm2 = static_cast<int>((d + kBM - 1) / kBM);
  p.glu = glu ? 1 : 0;
  p.kept_cnt = kept_cnt;
  p.H = static_cast<__nv_bfloat16*>(H);
  p.ye = static_cast<__nv_bfloat16*>(ye);
  p.tile_ctr = static_cast<unsigned int*>(sync);
  p.chunk_ctr = static_cast<unsigned int*>(sync) + 1;
  p.status = status;
  p.wait_ns = wait_limit_ns();
  if (top1) {
    p.tok_of_row = top1->tok_of_row;
    p.gate = top1->gate;
    p.y = static_cast<__nv_bfloat16*>(top1->y);
  }
  if (cudaFuncSetAttribute(ffn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSmemBytes) != cudaSuccess)
    return check_launch("cudaFuncSetAttribute(ffn_pair_kernel)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms() & ~1));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // cluster shape only, for the occupancy query
  int resident = 0;
  if (cudaOccupancyMaxActiveClusters(&resident, ffn_pair_kernel, &cfg) != cudaSuccess ||
      resident < 1)
    return check_launch("cudaOccupancyMaxActiveClusters(ffn_pair_kernel)");
  // lag: the GEMM-2 tiles of expert e come after the GEMM-1 tiles of the next
  // L experts, about three tiles per pair (each pair holds up to three tiles
  // between taking one and finishing its epilogue), so their wait for H is
  // normally over when they are taken; chunks per expert estimated as C / 256
  const int64_t g1_per_expert = std::max<int64_t>(1, static_cast<int64_t>(p.nm1) * C / kChunk);
  p.lag = static_cast<int>(std::min<int64_t>(
      E, std::max<int64_t>(1, (3 * static_cast<int64_t>(resident) + g1_per_expert - 1) /
                                  g1_per_expert)));
  const int64_t max_tiles = E * static_cast<int64_t>(maxc) * (p.nm1 + p.nm2);
  if (max_tiles > 2147483647) return fail(MOE_ERR_UNSUPPORTED, "ffn_pair_kernel: too many tiles");
  const int64_t clusters = std::min<int64_t>(resident, max_tiles);
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
  cfg.numAttrs = 2;
  cudaLaunchKernelEx(&cfg, ffn_pair_kernel, maps, p);
  return check_launch("ffn_pair_kernel");
}

}  // namespace moe
