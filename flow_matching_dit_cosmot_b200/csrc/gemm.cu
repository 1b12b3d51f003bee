// Routed projection GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "Cosmos 3 方法原理全解" §3: a MoT layer holds two weight sets; Reasoner
// weights act on AR rows and Generator weights on DM rows, with no router.
// Rows come in segments (a contiguous row range and its weight set); a tile
// never straddles two segments, so every tile runs one dense contraction
//     acc[128 x 256] = A[rows, K] . W_set[cols, K]^T
// on the tensor cores with the fp32 accumulator in tensor memory.
//
// Structure (one persistent CTA per SM, 192 threads; for most calls a pair of
// CTAs per 256-row tile, see Tiles below):
//   warp 0      TMA producer: A tile 128x64 and B tile 256x64 (bf16, 128-byte
//               swizzle) per k-block into a 4-stage shared-memory ring.
//   warp 1      owns TMEM (512 columns = two 128x256 fp32 accumulators) and
//               issues tcgen05.mma (M=128, N=256, K=16) from one thread;
//               tcgen05.commit frees ring slots and publishes accumulators.
//   warps 2-5   epilogue: tcgen05.ld (one row per thread), the fused
//               epilogue (residual add, SiLU*mul, mRoPE, Euler), bf16 stores.
// The epilogue of tile i overlaps the mainloop of tile i+1.  Tiles are walked
// in groups of kGroupM row tiles so that a group's A rows stay in L2 while the
// weight columns stream past.
//
// Every wait is bounded (see ptx.cuh): a stuck pipeline latches
// COSMOT_ERR_TIMEOUT, drains its outstanding copies and MMAs, frees TMEM and
// returns.
#include <cuda_bf16.h>

#include <mutex>

#include "cosmot_internal.h"
#include "ptx.cuh"

namespace cosmot {
namespace gemm {

constexpr int BM = 128;
constexpr int BK = 64;  // 64 bf16 = 128 bytes = one swizzle row
constexpr int A_BYTES = BM * BK * 2;
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 512;
constexpr int kMaxSegs = 64;
constexpr int kGroupM = 16;

// Tile width BN: 256 by default; 160 where a call has too few output tiles to
// fill the SMs with 256-wide ones (a few hundred rows against a 4096-wide
// output: 5 row tiles x 16 column tiles = 80 tiles for 148 SMs become 5 x 26
// = 130).  Any multiple of 32 up to 256 is a valid tcgen05 N for M = 128.
// Such calls read their weights cold, once, and wait on the loads, so tiles
// up to 160 wide keep six stages in flight (216 KB) where 256-wide ones fit
// four.
//
// CG = 2: a cluster of two CTAs computes a 256-row tile, 256 (or 224) columns
// wide, with tcgen05.mma.cta_group::2 (M = 256): each CTA loads its own 128 A
// rows and half of the B rows (the gate or the up half for SiLU*mul), so a
// CTA moves 32 KB per k-block instead of 48 KB for the same work, and six
// stages fit.  The even CTA's full barrier counts both CTAs' bytes; its MMA
// thread commits to both CTAs' barriers; both epilogues release an
// accumulator on the even CTA's barrier.  The tile plan (cosmot_routed_linear)
// keeps single-CTA tiles (CG = 1) for calls with a few hundred rows.
template <int BN, int CG = 1>
struct Tiles {
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "tile width");
  static_assert(CG == 1 || (CG == 2 && (BN == 256 || BN == 224)), "pair tiles are 256 x 256 or 256 x 224");
  static constexpr int STAGES = CG == 2 || BN <= 160 ? 6 : 4;
  static constexpr int B_BYTES = BN * BK * 2 / CG;  // this CTA's B rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 256 + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM * CG, BN, false, false);
};

struct Params {
  int64_t row_begin[kMaxSegs];
  int64_t row_end[kMaxSegs];
  int64_t out_row[kMaxSegs];
  int32_t set[kMaxSegs];
  int32_t mtile_prefix[kMaxSegs + 1];
  int32_t n_segs;
  int32_t num_m_tiles, num_n_tiles, num_tiles;
  int32_t num_kb;
  int32_t n_out;
  int32_t head_dim;
  int32_t group_m;
  int64_t rope_cols;
  const float2* rope_cs;
  int64_t rope_period;
  const void* res;        // bf16, or float32 with COSMOT_EPI_RES_F32
  int64_t ld_res;
  const __nv_bfloat16* x;
  int64_t ld_x;
  float dsigma;
  int32_t xs_from_x;      // EULER with xs: read x from the bf16 `x` this call
  float* xs;              // EULER: optional float32 state, indexed by input row
  int64_t ld_xs;
  __nv_bfloat16* vel;     // EULER: optional bf16 copy of the accumulator, by input row
  int64_t ld_vel;
  __nv_bfloat16* out;     // float32 storage with COSMOT_EPI_OUT_F32
  int64_t ld_out;
  int64_t out_rows;       // output rows the segments address (debug store checks)
  int64_t a_rows;         // input rows the segments address (x_state / vel rows)
  int* status;
};

struct Tile {
  int32_t set;
  int32_t n;          // column tile
  int64_t a_row0;     // first A row
  int32_t rows;       // valid rows (<= the tile's rows)
  int64_t out_row0;   // output row of a_row0
};

// TM: rows of a tile (128, or 256 for a pair of CTAs).
template <int TM>
__device__ __forceinline__ Tile decode_tile(const Params& p, int32_t t) {
  const int32_t per_group = p.group_m * p.num_n_tiles;
  const int32_t g = t / per_group;
  const int32_t first_m = g * p.group_m;
  const int32_t rem_m = p.num_m_tiles - first_m;
  const int32_t gm = rem_m < p.group_m ? rem_m : p.group_m;
  const int32_t in = t - g * per_group;
  const int32_t m = first_m + in % gm;
  Tile tl;
  tl.n = in / gm;
  int s = 0;
  while (s + 1 < p.n_segs && m >= p.mtile_prefix[s + 1]) ++s;
  tl.set = p.set[s];
  tl.a_row0 = p.row_begin[s] + (int64_t)(m - p.mtile_prefix[s]) * TM;
  const int64_t left = p.row_end[s] - tl.a_row0;
  tl.rows = (int32_t)(left < TM ? left : TM);
  tl.out_row0 = p.out_row[s] + (tl.a_row0 - p.row_begin[s]);
  return tl;
}

// Stores 32 consecutive fp32 values of one row as bf16, clipped to n_out.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, int32_t col0, int32_t n_out, const float* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (col0 + 8 * q + 8 <= n_out) {
      uint4 w;
      w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
      w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
      w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
      w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
      *reinterpret_cast<uint4*>(dst + 8 * q) = w;
    }
  }
}

// Stores / loads 32 consecutive fp32 values of one row, clipped to n_out.
__device__ __forceinline__ void store_row32_f32(float* dst, int32_t col0, int32_t n_out, const float* v) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    if (col0 + 4 * q + 4 <= n_out)
      *reinterpret_cast<float4*>(dst + 4 * q) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

__device__ __forceinline__ void load_row32_f32(const float* src, int32_t col0, int32_t n_out, float* v) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
    if (col0 + 4 * q + 4 <= n_out) w = *reinterpret_cast<const float4*>(src + 4 * q);
    v[4 * q] = w.x;
    v[4 * q + 1] = w.y;
    v[4 * q + 2] = w.z;
    v[4 * q + 3] = w.w;
  }
}

// Loads 32 consecutive bf16 of one row as fp32 (zeros past n_out).
__device__ __forceinline__ void load_row32(const __nv_bfloat16* src, int32_t col0, int32_t n_out, float* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (col0 + 8 * q + 8 <= n_out) {
      uint4 w = *reinterpret_cast<const uint4*>(src + 8 * q);
      const uint32_t* u = reinterpret_cast<const uint32_t*>(&w);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 f = unpack_bf16x2(u[j]);
        v[8 * q + 2 * j] = f.x;
        v[8 * q + 2 * j + 1] = f.y;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[8 * q + j] = 0.f;
    }
  }
}

// FL: COSMOT_EPI_OUT_F32 / COSMOT_EPI_RES_F32 bits of the RESIDUAL epilogue;
// BN: the tile width; CG: CTAs per tile (2: launched as clusters of two).
template <int EPI, int FL, int BN, int CG>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    routed_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b0,
                       const __grid_constant__ CUtensorMap tmap_b1, const __grid_constant__ CUtensorMap tmap_u0,
                       const __grid_constant__ CUtensorMap tmap_u1, const __grid_constant__ Params p) {
  using T = Tiles<BN, CG>;
  constexpr int STAGES = T::STAGES;
  constexpr int B_BYTES = T::B_BYTES;
  constexpr int STAGE_BYTES = T::STAGE_BYTES;
  constexpr uint32_t IDESC = T::IDESC;
  constexpr int TM = BM * CG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  const uint32_t bar_full = smem_u32(bars);                // [STAGES]
  const uint32_t bar_empty = bar_full + 8 * STAGES;        // [STAGES]
  const uint32_t bar_tfull = bar_empty + 8 * STAGES;       // [2]
  const uint32_t bar_tempty = bar_tfull + 16;              // [2]
  const uint32_t bar_drain = bar_tempty + 16;              // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Pair tiles: `rank` 0 (even CTA) issues the MMAs; tile work is walked per pair.
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const int32_t unit = CG == 2 ? (int32_t)(blockIdx.x >> 1) : (int32_t)blockIdx.x;
  const int32_t units = CG == 2 ? (int32_t)(gridDim.x >> 1) : (int32_t)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_tfull + 8 * b, 1);
      // one arrive per epilogue thread; pairs: one per epilogue warp of both CTAs
      mbar_init(bar_tempty + 8 * b, CG == 2 ? 8 : 4 * 32);
    }
    mbar_init(bar_drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (CG == 2) {
      tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (CG == 2) cluster_sync();  // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b0);
    tma_prefetch_desc(&tmap_b1);
    if (EPI == COSMOT_EPI_SILU_MUL) {
      tma_prefetch_desc(&tmap_u0);
      tma_prefetch_desc(&tmap_u1);
    }
  }
  // Up to here the CTA touched only its own shared and tensor memory and the
  // kernel parameters, so this prologue may overlap the previous kernel.
  pdl_trigger();
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed_mask = 0, armed_parity = 0;
      bool ok = true;
      for (int32_t t = unit; t < p.num_tiles && ok; t += units) {
        const Tile tl = decode_tile<TM>(p, t);
        const CUtensorMap* mb = tl.set ? &tmap_b1 : &tmap_b0;
        const CUtensorMap* mu = tl.set ? &tmap_u1 : &tmap_u0;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, p.status, kWhereGemmProducer)) {
            ok = false;
            break;
          }
          const uint32_t fb = bar_full + 8 * stage;
          const uint32_t sa = sbase + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          if constexpr (CG == 2) {
            // both CTAs' bytes complete on the even CTA's barrier, which only it arms
            const uint32_t fb0 = mapa_shared(fb, 0);
            if (rank == 0) mbar_arrive_expect_tx(fb, 2 * STAGE_BYTES);
            tma_load_2d_pair(sa, &tmap_a, fb0, kb * BK, (int)(tl.a_row0 + (int64_t)rank * BM));
            if (EPI == COSMOT_EPI_SILU_MUL)
              tma_load_2d_pair(sb, rank ? mu : mb, fb0, kb * BK, tl.n * (BN / 2));
            else
              tma_load_2d_pair(sb, mb, fb0, kb * BK, tl.n * BN + (int)rank * (BN / 2));
          } else {
            mbar_arrive_expect_tx(fb, STAGE_BYTES);
            tma_load_2d(sa, &tmap_a, fb, kb * BK, (int)tl.a_row0);
            if (EPI == COSMOT_EPI_SILU_MUL) {
              tma_load_2d(sb, mb, fb, kb * BK, tl.n * (BN / 2));
              tma_load_2d(sb + B_BYTES / 2, mu, fb, kb * BK, tl.n * (BN / 2));
            } else {
              tma_load_2d(sb, mb, fb, kb * BK, tl.n * BN);
            }
          }
          armed_mask |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // No bulk copy may still be writing shared memory when the CTA exits.
      // Pairs: the even CTA's barriers count the odd CTA's copies too, and the
      // odd CTA leaves only after the closing cluster barrier.
      for (int s = 0; s < STAGES; ++s)
        if (rank == 0 && (armed_mask & (1u << s))) {
          const uint32_t par = (armed_parity >> s) & 1u;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(bar_full + 8 * s, par) && globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t local = 0;
      for (int32_t t = unit; t < p.num_tiles && ok; t += units, ++local) {
        const uint32_t buf = local & 1;
        const uint32_t use = local >> 1;
        if (!mbar_wait(bar_tempty + 8 * buf, (use & 1) ^ 1, p.status, kWhereGemmMma)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(bar_full + 8 * stage, phase, p.status, kWhereGemmMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = sw128_desc(sa + 32 * k, 16, 1024);
            const uint64_t bd = sw128_desc(sb + 32 * k, 16, 1024);
            if constexpr (CG == 2)
              umma_ss_pair(d_tmem, ad, bd, IDESC, (kb | k) != 0 ? 1u : 0u);
            else
              umma_ss(d_tmem, ad, bd, IDESC, (kb | k) != 0 ? 1u : 0u);
          }
          if constexpr (CG == 2)
            umma_commit_pair_mc(bar_empty + 8 * stage, 3);
          else
            umma_commit(bar_empty + 8 * stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if constexpr (CG == 2)
          umma_commit_pair_mc(bar_tfull + 8 * buf, 3);
        else
          umma_commit(bar_tfull + 8 * buf);
      }
      // Wait until every MMA issued above has completed before TMEM is freed.
      if constexpr (CG == 2)
        umma_commit_pair_mc(bar_drain, 1);
      else
        umma_commit(bar_drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar_drain, 0)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          latch_status(p.status, COSMOT_ERR_TIMEOUT, kWhereGemmDrain);
          break;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int lane_base = (warp & 3) * 32;  // TMEM lanes this warp may access
    const int r = lane_base + lane;          // row within the tile
    uint32_t local = 0;
    for (int32_t t = unit; t < p.num_tiles; t += units, ++local) {
      const uint32_t buf = local & 1;
      const uint32_t use = local >> 1;
      // Warp-uniform: the tcgen05.ld below is .sync.aligned.
      if (!__all_sync(0xffffffffu, mbar_wait(bar_tfull + 8 * buf, use & 1, p.status, kWhereGemmEpilogue))) break;
      tc_fence_after();
      const Tile tl = decode_tile<TM>(p, t);
      const int rr = (int)rank * BM + r;  // row within the (pair's) tile
      const bool valid = rr < tl.rows;
      const int64_t orow = tl.out_row0 + rr;
      const uint32_t tacc = tmem_base + ((uint32_t)lane_base << 16) + buf * BN;
      uint32_t v[32];
      float f[32];
      if (EPI == COSMOT_EPI_SILU_MUL) {
        const int32_t col_base = tl.n * (BN / 2);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t u[32];
          tmem_ld32(tacc + 32 * c, v);
          tmem_ld32(tacc + BN / 2 + 32 * c, u);
          tmem_ld_wait();
          const int32_t col0 = col_base + 32 * c;
          if (valid && col0 < p.n_out && dcheck(orow >= 0 && orow < p.out_rows, p.status, kWhereGemmStore)) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float g = __uint_as_float(v[j]);
              const float up = __uint_as_float(u[j]);
              f[j] = g / (1.0f + __expf(-g)) * up;
            }
            store_row32(p.out + orow * p.ld_out + col0, col0, p.n_out, f);
          }
        }
      } else if (EPI == COSMOT_EPI_MROPE) {
        const int hd = p.head_dim;
        const int half = hd >> 1;
        const int64_t arow = tl.a_row0 + rr;  // positions follow the input row
        const int64_t trow = p.rope_period > 0 ? arow % p.rope_period : arow;
        const float2* cs_row = p.rope_cs + trow * half;
#pragma unroll 1
        for (int hb = 0; hb < BN / hd; ++hb) {
          const int32_t hcol = tl.n * BN + hb * hd;
          const bool rotate = hcol < p.rope_cols;
#pragma unroll 1
          for (int i0 = 0; i0 < half; i0 += 32) {
            // the row's (cos, sin) of pairs i0 .. i0 + 31, requested before the
            // accumulator loads so that their latency overlaps
            float4 csv[16];
            if (valid && rotate) {
#pragma unroll
              for (int j = 0; j < 16; ++j) csv[j] = __ldg(reinterpret_cast<const float4*>(cs_row + i0 + 2 * j));
            }
            uint32_t u[32];
            tmem_ld32(tacc + hb * hd + i0, v);
            tmem_ld32(tacc + hb * hd + half + i0, u);
            tmem_ld_wait();
            if (valid && hcol < p.n_out && dcheck(orow >= 0 && orow < p.out_rows, p.status, kWhereGemmStore)) {
              float lo[32], hi[32];
              if (rotate) {
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                  const float4 cs = csv[j >> 1];
                  const float a0 = __uint_as_float(v[j]), a1 = __uint_as_float(v[j + 1]);
                  const float b0 = __uint_as_float(u[j]), b1 = __uint_as_float(u[j + 1]);
                  lo[j] = a0 * cs.x - b0 * cs.y;
                  hi[j] = b0 * cs.x + a0 * cs.y;
                  lo[j + 1] = a1 * cs.z - b1 * cs.w;
                  hi[j + 1] = b1 * cs.z + a1 * cs.w;
                }
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                  lo[j] = __uint_as_float(v[j]);
                  hi[j] = __uint_as_float(u[j]);
                }
              }
              __nv_bfloat16* dst = p.out + orow * p.ld_out + hcol;
              store_row32(dst + i0, hcol + i0, p.n_out, lo);
              store_row32(dst + half + i0, hcol + half + i0, p.n_out, hi);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          tmem_ld32(tacc + 32 * c, v);
          tmem_ld_wait();
          const int32_t col0 = tl.n * BN + 32 * c;
          if (valid && col0 < p.n_out && dcheck(orow >= 0 && orow < p.out_rows, p.status, kWhereGemmStore)) {
            if (EPI == COSMOT_EPI_RESIDUAL) {
              float rs[32];
              if (FL & COSMOT_EPI_RES_F32)
                load_row32_f32(static_cast<const float*>(p.res) + orow * p.ld_res + col0, col0, p.n_out, rs);
              else
                load_row32(static_cast<const __nv_bfloat16*>(p.res) + orow * p.ld_res + col0, col0, p.n_out, rs);
#pragma unroll
              for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]) + rs[j];
            } else if (EPI == COSMOT_EPI_EULER) {
              // x' = x + dsigma * v in fp32; x from the fp32 state when there is one
              const int64_t arow = tl.a_row0 + rr;
              const bool arow_ok = dcheck(arow >= 0 && arow < p.a_rows, p.status, kWhereGemmStore);
              float xs[32];
              if (p.xs && !p.xs_from_x && arow_ok)
                load_row32_f32(p.xs + arow * p.ld_xs + col0, col0, p.n_out, xs);
              else
                load_row32(p.x + orow * p.ld_x + col0, col0, p.n_out, xs);
#pragma unroll
              for (int j = 0; j < 32; ++j) f[j] = fmaf(p.dsigma, __uint_as_float(v[j]), xs[j]);
              if (p.xs && arow_ok) store_row32_f32(p.xs + arow * p.ld_xs + col0, col0, p.n_out, f);
              if (p.vel && arow_ok) {
                float vv[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) vv[j] = __uint_as_float(v[j]);
                store_row32(p.vel + arow * p.ld_vel + col0, col0, p.n_out, vv);
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]);
            }
            if (FL & COSMOT_EPI_OUT_F32)
              store_row32_f32(reinterpret_cast<float*>(p.out) + orow * p.ld_out + col0, col0, p.n_out, f);
            else
              store_row32(p.out + orow * p.ld_out + col0, col0, p.n_out, f);
          }
        }
      }
      tc_fence_before();
      if constexpr (CG == 2) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(bar_tempty + 8 * buf, 0));
      } else {
        mbar_arrive(bar_tempty + 8 * buf);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (CG == 2) cluster_sync();  // the pair's MMAs have drained; neither CTA's memory is in use
  tc_fence_after();
  if (warp == 1) {
    if constexpr (CG == 2)
      tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else
      tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// Clusters of two this kernel keeps resident at once on the current device
// (0 if it cannot run as pairs).
int resident_pairs() {
  static std::mutex mu;
  static int cached[64] = {0};
  static uint64_t done_mask = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lk(mu);
  if (!(done_mask & (1ull << dev))) {
    auto kern = routed_gemm_kernel<COSMOT_EPI_NONE, 0, 256, 2>;  // every pair instance has this footprint
    int n = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Tiles<256, 2>::SMEM_BYTES) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg{};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * 74, 1, 1);
      cfg.blockDim = dim3(NUM_THREADS, 1, 1);
      cfg.dynamicSmemBytes = Tiles<256, 2>::SMEM_BYTES;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
    }
    (void)cudaGetLastError();
    cached[dev] = n;
    done_mask |= 1ull << dev;
  }
  return cached[dev];
}

template <int EPI, int FL = 0, int BN = 256, int CG = 1>
cosmot_status launch(const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1, const CUtensorMap& tu0,
                     const CUtensorMap& tu1, const Params& p, cudaStream_t s) {
  constexpr int SMEM_BYTES = Tiles<BN, CG>::SMEM_BYTES;
  static std::mutex mu;
  static uint64_t done_mask = 0;  // devices whose smem limit was raised
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return COSMOT_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 64 || !(done_mask & (1ull << dev))) {
      if (cudaFuncSetAttribute(routed_gemm_kernel<EPI, FL, BN, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SMEM_BYTES) !=
          cudaSuccess)
        return COSMOT_ERR_CUDA;
      if (dev < 64) done_mask |= 1ull << dev;
    }
  }
  if constexpr (CG == 2) {
    int pairs = resident_pairs();
    if (pairs < 1) return COSMOT_ERR_CUDA;
    if (p.num_tiles < pairs) pairs = p.num_tiles;
    cudaLaunchAttribute cluster;
    cluster.id = cudaLaunchAttributeClusterDimension;
    cluster.val.clusterDim.x = 2;
    cluster.val.clusterDim.y = 1;
    cluster.val.clusterDim.z = 1;
    return launch_status(launch_pdl(routed_gemm_kernel<EPI, FL, BN, CG>, dim3(2 * pairs), dim3(NUM_THREADS), SMEM_BYTES,
                                    s, &cluster, ta, tb0, tb1, tu0, tu1, p));
  }
  int grid = num_sms();
  if (p.num_tiles < grid) grid = p.num_tiles;
  return launch_status(launch_pdl(routed_gemm_kernel<EPI, FL, BN, CG>, dim3(grid), dim3(NUM_THREADS), SMEM_BYTES, s,
                                  nullptr, ta, tb0, tb1, tu0, tu1, p));
}

}  // namespace gemm
}  // namespace cosmot

extern "C" cosmot_status cosmot_routed_linear(const void* a, int64_t ld_a, int64_t k, const cosmot_segment* segs,
                                              int32_t n_segs, const void* w0, const void* w1, const void* w0_up,
                                              const void* w1_up, int64_t n_out, void* out, int64_t ld_out,
                                              const cosmot_epilogue* epi, cosmot_stream_t stream) {
  using namespace cosmot;
  using namespace cosmot::gemm;
  const int kind = epi ? epi->kind : COSMOT_EPI_NONE;
  if (!a || !out || !segs || n_segs < 1 || n_segs > kMaxSegs) return COSMOT_ERR_INVALID_ARG;
  if (k < 8 || k % 8 || n_out < 8 || n_out % 8 || ld_a % 8 || ld_out % 8 || ld_a < k || ld_out < n_out)
    return COSMOT_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(out)) return COSMOT_ERR_INVALID_ARG;
  if (k > INT32_MAX || n_out > INT32_MAX) return COSMOT_ERR_UNSUPPORTED;
  if (kind < COSMOT_EPI_NONE || kind > COSMOT_EPI_EULER) return COSMOT_ERR_INVALID_ARG;
  const int flags = epi ? epi->flags : 0;
  if (flags & ~(COSMOT_EPI_OUT_F32 | COSMOT_EPI_RES_F32)) return COSMOT_ERR_INVALID_ARG;
  if (flags && kind != COSMOT_EPI_RESIDUAL) return COSMOT_ERR_INVALID_ARG;

  Params p{};
  p.n_segs = n_segs;
  bool uses[2] = {false, false};
  int64_t max_row = 0;
  for (int i = 0; i < n_segs; ++i) {
    const cosmot_segment& s = segs[i];
    if (s.row_begin < 0 || s.row_end < s.row_begin || s.out_row < 0 || (s.weight_set != 0 && s.weight_set != 1))
      return COSMOT_ERR_INVALID_ARG;
    if (s.row_end - s.row_begin > INT32_MAX / 4) return COSMOT_ERR_UNSUPPORTED;
    p.row_begin[i] = s.row_begin;
    p.row_end[i] = s.row_end;
    p.out_row[i] = s.out_row;
    p.set[i] = s.weight_set;
    if (s.row_end > s.row_begin) uses[s.weight_set] = true;
    if (s.row_end > max_row) max_row = s.row_end;
  }
  // row tiles of `tm` rows over all segments (a tile never straddles two)
  auto count_mtiles = [&](int64_t tm) {
    int64_t n = 0;
    for (int i = 0; i < n_segs; ++i) n += (segs[i].row_end - segs[i].row_begin + tm - 1) / tm;
    return n;
  };
  const int64_t mt1 = count_mtiles(BM);
  if (mt1 > INT32_MAX / 4) return COSMOT_ERR_UNSUPPORTED;
  const int32_t mt = (int32_t)mt1;
  for (int i = 0; i < n_segs; ++i) {
    const int64_t end = segs[i].out_row + (segs[i].row_end - segs[i].row_begin);
    if (end > p.out_rows) p.out_rows = end;
  }
  p.a_rows = max_row;
  if (mt == 0) return COSMOT_OK;
  const int64_t sms = num_sms();
  auto rounds = [](int64_t tiles, int64_t slots) { return (tiles + slots - 1) / slots; };
  if (max_row > INT32_MAX) return COSMOT_ERR_UNSUPPORTED;
  const bool silu = kind == COSMOT_EPI_SILU_MUL;
  // Tile width: 160 instead of 256 when that keeps clearly more SMs busy over
  // the waves of tiles (mRoPE needs whole heads in a tile, SiLU*mul a gate and
  // an up half: both keep 256).
  int bn = 256;
  if (kind == COSMOT_EPI_NONE || kind == COSMOT_EPI_RESIDUAL || kind == COSMOT_EPI_EULER) {
    auto eff = [&](int64_t w) {
      const int64_t t = (int64_t)mt * ((n_out + w - 1) / w);
      return (double)t / (double)(((t + sms - 1) / sms) * sms);
    };
    if (eff(160) > eff(256) + 0.1) bn = 160;
  }
  p.num_n_tiles = (int32_t)((n_out + (silu ? bn / 2 : bn) - 1) / (silu ? bn / 2 : bn));
  // CTA pairs (256-row tiles, half the B bytes a CTA) when their rounds over
  // the SMs, times the tile width, cost no more than single-CTA tiles' with a
  // 20 % surcharge for the single-CTA main loop's load waits (a clock64
  // trace: 20-25 % of each tile against 12 % for pairs).  Pairs are 256 or
  // 224 columns wide (224 fills the last round better at a few thousand
  // rows; mRoPE and SiLU*mul keep 256).  On the 480p layer pairs took QKV
  // from 1.49 to 1.38 ms and the O projection from 0.57 to 0.50 ms.
  int cg = 1;
  {
    const int64_t pairs = resident_pairs();
    if (pairs > 0) {
      const int64_t cost1 = rounds(mt1 * p.num_n_tiles, sms) * bn * 6;  // x 5, plus the 20 %
      const int64_t mt2 = count_mtiles(2 * BM);
      const bool narrow_ok = kind == COSMOT_EPI_NONE || kind == COSMOT_EPI_RESIDUAL || kind == COSMOT_EPI_EULER;
      int best = 0;
      int64_t best_cost = cost1;
      for (int w : {256, 224}) {
        if (w != 256 && !narrow_ok) continue;
        const int64_t cols = silu ? w / 2 : w;
        const int64_t cost = rounds(mt2 * ((n_out + cols - 1) / cols), pairs) * w * 5;
        if (cost <= best_cost) {
          best_cost = cost;
          best = w;
        }
      }
      if (best) {
        cg = 2;
        bn = best;
        p.num_n_tiles = (int32_t)((n_out + (silu ? bn / 2 : bn) - 1) / (silu ? bn / 2 : bn));
      }
    }
  }
  const int64_t tm = (int64_t)BM * cg;
  int32_t mtc = 0;
  for (int i = 0; i < n_segs; ++i) {
    p.mtile_prefix[i] = mtc;
    mtc += (int32_t)((segs[i].row_end - segs[i].row_begin + tm - 1) / tm);
  }
  p.mtile_prefix[n_segs] = mtc;
  p.num_m_tiles = mtc;
  if ((int64_t)p.num_m_tiles * p.num_n_tiles > INT32_MAX) return COSMOT_ERR_UNSUPPORTED;
  p.num_tiles = p.num_m_tiles * p.num_n_tiles;
  p.num_kb = (int32_t)((k + BK - 1) / BK);
  p.n_out = (int32_t)n_out;
  p.group_m = kGroupM / cg;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.ld_out = ld_out;
  p.status = device_status_ptr();
  if (!p.status) return COSMOT_ERR_CUDA;

  if (kind == COSMOT_EPI_RESIDUAL) {
    if (!epi->res || !aligned16(epi->res) || epi->ld_res % 8 || epi->ld_res < n_out) return COSMOT_ERR_INVALID_ARG;
    p.res = epi->res;
    p.ld_res = epi->ld_res;
  } else if (kind == COSMOT_EPI_EULER) {
    if (!epi->x || !aligned16(epi->x) || epi->ld_x % 8 || epi->ld_x < n_out) return COSMOT_ERR_INVALID_ARG;
    p.x = static_cast<const __nv_bfloat16*>(epi->x);
    p.ld_x = epi->ld_x;
    p.dsigma = epi->dsigma;
    if (epi->x_state) {
      if (!aligned16(epi->x_state) || epi->ld_state % 8 || epi->ld_state < n_out) return COSMOT_ERR_INVALID_ARG;
      p.xs = epi->x_state;
      p.ld_xs = epi->ld_state;
      p.xs_from_x = epi->state_from_x ? 1 : 0;
    }
    if (epi->vel) {
      if (!aligned16(epi->vel) || epi->ld_vel % 8 || epi->ld_vel < n_out) return COSMOT_ERR_INVALID_ARG;
      p.vel = static_cast<__nv_bfloat16*>(epi->vel);
      p.ld_vel = epi->ld_vel;
    }
  } else if (kind == COSMOT_EPI_MROPE) {
    if (epi->head_dim != 64 && epi->head_dim != 128) return COSMOT_ERR_UNSUPPORTED;
    if (!epi->rope_cs || !aligned16(epi->rope_cs) || epi->rope_cols < 0 || epi->rope_cols % epi->head_dim ||
        epi->rope_cols > n_out || epi->rope_period < 0)
      return COSMOT_ERR_INVALID_ARG;
    p.head_dim = epi->head_dim;
    p.rope_cols = epi->rope_cols;
    p.rope_cs = reinterpret_cast<const float2*>(epi->rope_cs);
    p.rope_period = epi->rope_period;
  }

  // Tensor maps: A over all rows the segments touch; B per weight set.
  CUtensorMap ta, tb[2], tu[2];
  cosmot_status st = make_tmap_bf16_2d(&ta, a, (uint64_t)max_row, (uint64_t)k, (uint64_t)ld_a, BM, BK);
  if (st != COSMOT_OK) return st;
  const void* wb[2] = {w0, w1};
  const void* wu[2] = {w0_up, w1_up};
  // a CTA's B box: the tile's columns, the gate or up half for SiLU*mul, and
  // for a pair of CTAs one half of either
  const uint32_t brows = cg == 2 ? (uint32_t)bn / 2 : (silu ? bn / 2 : bn);
  for (int s = 0; s < 2; ++s) {
    const int src = uses[s] ? s : (uses[0] ? 0 : 1);  // an unused set reuses a valid map
    if (!wb[src]) return COSMOT_ERR_INVALID_ARG;
    st = make_tmap_bf16_2d(&tb[s], wb[src], (uint64_t)n_out, (uint64_t)k, (uint64_t)k, brows, BK);
    if (st != COSMOT_OK) return st;
    if (silu) {
      if (!wu[src]) return COSMOT_ERR_INVALID_ARG;
      st = make_tmap_bf16_2d(&tu[s], wu[src], (uint64_t)n_out, (uint64_t)k, (uint64_t)k, brows, BK);
      if (st != COSMOT_OK) return st;
    } else {
      tu[s] = tb[s];
    }
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cg == 2 && bn == 224) {
    switch (kind) {
      case COSMOT_EPI_NONE: return launch<COSMOT_EPI_NONE, 0, 224, 2>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
      case COSMOT_EPI_EULER: return launch<COSMOT_EPI_EULER, 0, 224, 2>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
      default:
        switch (flags) {
          case COSMOT_EPI_OUT_F32:
            return launch<COSMOT_EPI_RESIDUAL, COSMOT_EPI_OUT_F32, 224, 2>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
          case COSMOT_EPI_RES_F32:
            return launch<COSMOT_EPI_RESIDUAL, COSMOT_EPI_RES_F32, 224, 2>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
          case COSMOT_EPI_OUT_F32 | COSMOT_EPI_RES_F32:
            return launch<COSMOT_EPI_RESIDUAL, COSMOT_EPI_OUT_F32 | COSMOT_EPI_RES_F32, 224, 2>(ta, tb[0], tb[1], tu[0],
                                                                                              tu[1], p, s);
          default: return launch<COSMOT_EPI_RESIDUAL, 0, 224, 2>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
        }
    }
  }
  if (cg == 2) {
    switch (kind) {
      case COSMOT_EPI_NONE: return launch<COSMOT_EPI_NONE, 0, 256, 2>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
      case COSMOT_EPI_SILU_MUL: return launch<COSMOT_EPI_SILU_MUL, 0, 256, 2>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
      case COSMOT_EPI_MROPE: return launch<COSMOT_EPI_MROPE, 0, 256, 2>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
      case COSMOT_EPI_EULER: return launch<COSMOT_EPI_EULER, 0, 256, 2>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
      default:
        switch (flags) {
          case COSMOT_EPI_OUT_F32:
            return launch<COSMOT_EPI_RESIDUAL, COSMOT_EPI_OUT_F32, 256, 2>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
          case COSMOT_EPI_RES_F32:
            return launch<COSMOT_EPI_RESIDUAL, COSMOT_EPI_RES_F32, 256, 2>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
          case COSMOT_EPI_OUT_F32 | COSMOT_EPI_RES_F32:
            return launch<COSMOT_EPI_RESIDUAL, COSMOT_EPI_OUT_F32 | COSMOT_EPI_RES_F32, 256, 2>(ta, tb[0], tb[1], tu[0],
                                                                                              tu[1], p, s);
          default: return launch<COSMOT_EPI_RESIDUAL, 0, 256, 2>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
        }
    }
  }
  if (bn == 160) {
    switch (kind) {
      case COSMOT_EPI_NONE: return launch<COSMOT_EPI_NONE, 0, 160>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
      case COSMOT_EPI_EULER: return launch<COSMOT_EPI_EULER, 0, 160>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
      default:
        switch (flags) {
          case COSMOT_EPI_OUT_F32:
            return launch<COSMOT_EPI_RESIDUAL, COSMOT_EPI_OUT_F32, 160>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
          case COSMOT_EPI_RES_F32:
            return launch<COSMOT_EPI_RESIDUAL, COSMOT_EPI_RES_F32, 160>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
          case COSMOT_EPI_OUT_F32 | COSMOT_EPI_RES_F32:
            return launch<COSMOT_EPI_RESIDUAL, COSMOT_EPI_OUT_F32 | COSMOT_EPI_RES_F32, 160>(ta, tb[0], tb[1], tu[0],
                                                                                          tu[1], p, s);
          default: return launch<COSMOT_EPI_RESIDUAL, 0, 160>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
        }
    }
  }
  switch (kind) {
    case COSMOT_EPI_NONE: return launch<COSMOT_EPI_NONE>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
    case COSMOT_EPI_RESIDUAL:
      switch (flags) {
        case COSMOT_EPI_OUT_F32: return launch<COSMOT_EPI_RESIDUAL, COSMOT_EPI_OUT_F32>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
        case COSMOT_EPI_RES_F32: return launch<COSMOT_EPI_RESIDUAL, COSMOT_EPI_RES_F32>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
        case COSMOT_EPI_OUT_F32 | COSMOT_EPI_RES_F32:
          return launch<COSMOT_EPI_RESIDUAL, COSMOT_EPI_OUT_F32 | COSMOT_EPI_RES_F32>(ta, tb[0], tb[1], tu[0], tu[1],
                                                                                     p, s);
        default: return launch<COSMOT_EPI_RESIDUAL>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
      }
    case COSMOT_EPI_SILU_MUL: return launch<COSMOT_EPI_SILU_MUL>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
    case COSMOT_EPI_MROPE: return launch<COSMOT_EPI_MROPE>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
    default: return launch<COSMOT_EPI_EULER>(ta, tb[0], tb[1], tu[0], tu[1], p, s);
  }
}
