// MoT attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "Cosmos 3 方法原理全解" §3:
//     O_AR = Attn_causal(Q_AR, K_AR, V_AR)
//     O_DM = Attn_full(Q_DM, [K_AR; K_DM], [V_AR; V_DM])
// plus the time-causal block variant of "流式生成如何工作" (DM keys of later
// chunks hidden).  Softmax is the usual online (running max / running sum)
// formulation, exact up to rounding.
//
// One CTA per (sequence, head, pair of 128-row query tiles); a pair never
// mixes AR and DM rows.  384 threads in three warpgroups:
//   warp 0      TMA: both Q tiles once, then K_j and V_j tiles (128 keys x
//               head_dim, 128-byte swizzle) through a 4-slot ring.
//   warp 1      owns TMEM and issues the MMAs from one thread:
//                 S_t = Q_t K_j^T          (M=128, N=128, K=head_dim; SS)
//                 O_t += P_t V_j           (M=128, N=head_dim, K=128;  A = P in TMEM)
//               in the order S0 S1 | PV0 S0' PV1 S1' | ..., so the tensor core
//               works on one tile while the other tile's softmax runs.
//   warps 2-3   idle: they complete warpgroup 0, which hands registers to
//               the softmax (setmaxnreg: 88 a thread for warpgroup 0, 200 for
//               warpgroups 1 and 2, out of the 168 a thread at launch).
//   warps 4-7   softmax of query tile 0, warps 8-11 of tile 1 (one row per
//               thread): read S from TMEM, mask, running max, P = 2^(s*c - m)
//               written back over S as packed bf16, running sum; O is
//               rescaled in TMEM only when the running max grows by more than
//               2^8 (the exponent headroom keeps P and O finite meanwhile).
// TMEM columns: S0 [0,128), S1 [128,256), O0 and O1 after them.
//
// P is released in two halves (keys 0-63, then 64-127) so that the first half
// of PV overlaps the exponentials of the second; each softmax warp signals a
// half with one arrive after its lanes' tensor-memory stores have completed.
//
// Measured on B200 (18,978 tokens, 32 heads of 128): the period of one key
// block (~3,600 cycles before the register hand-over) is the chain
// softmax(tile 0) ~1,900 -> hand-off ~450 -> PV0 rest and next S0 ~1,000 ->
// S-ready ~250.  The softmax was held back by the 168-register ceiling of a
// CTA this size: giving it 200 registers a thread took the kernel from 5.6 to
// 5.1 ms on one box (tensor pipe 54 -> 59 %, SFU 54 -> 60 %).  It is bound by
// its own issue latency (one warp per sub-partition per tile), not by the SFU:
// exponentials on the FMA pipe (25 % or 37.5 % of them), packed f32x2
// arithmetic, a row split between two warpgroups, one warpgroup serving both
// tiles, and starting the exponentials of keys 0-63 from the previous running
// max while the tile max is reduced were all slower.  Smaller MMAs
// do not help either: a tcgen05.mma with N = 64 costs 44-48 cycles instead of
// 32 (fixed per-instruction cost), so 64-key blocks with double-buffered S, or
// S issued as two N = 64 halves, were 23-58 % slower.  Every tcgen05.ld/st is
// reached through warp-uniform control flow (they are .sync.aligned).
#include <cuda_bf16.h>

#include <mutex>

#include "cosmot_internal.h"
#include "ptx.cuh"

namespace cosmot {
namespace attn {

constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int SLOTS = 4;
constexpr int BOX_BYTES = 128 * 64 * 2;  // one 128-row x 64-column bf16 box
constexpr int NUM_THREADS = 384;
// Registers a thread after the hand-over; 128 x kRegsIo + 256 x kRegsSoftmax
// must not exceed the launch's pool (384 x registers at launch), or the
// increase would wait forever: the launch checks it.
constexpr int kRegsIo = 88;
constexpr int kRegsSoftmax = 200;
constexpr int TMEM_COLS = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Block-causal DM work items skip key tiles that none of their rows sees; the
// visit list is a bitmask in shared memory (one bit per 128-key tile).
constexpr int kMaxVisitWords = 2048;
constexpr int64_t kMaxVisitTiles = (int64_t)kMaxVisitWords * 32;
constexpr int32_t kMaxKvSplit = 8;

template <int HD>
struct Cfg {
  static constexpr int NBOX = HD / 64;
  static constexpr int TILE_BYTES = 128 * HD * 2;
  static constexpr int SMEM_BYTES = (2 + SLOTS) * TILE_BYTES + 256 + 4 * kMaxVisitWords + 1024;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BQ, BKV, false, false);
  static constexpr uint32_t IDESC_O = idesc_bf16_f32(BQ, HD, false, true);
  __device__ static constexpr uint32_t s_col(int t) { return (uint32_t)t * 128u; }
  __device__ static constexpr uint32_t o_col(int t) { return 256u + (uint32_t)t * HD; }
};

struct Params {
  int64_t n_q, q_key_offset, n_keys, n_ar;
  int64_t n_q_ar;  // leading query rows that are AR
  int64_t q_bstride, kv_bstride, o_bstride;
  int32_t n_heads, group;  // group = n_heads / n_kv_heads
  int32_t mask_mode;
  int32_t batch;
  int32_t dm_pairs, ar_pairs;
  int32_t skip;  // block-causal DM items skip key tiles none of their rows sees
  float scale_log2;
  const int32_t* chunk;
  __nv_bfloat16* o;
  int64_t ld_o;
  // Key split of the DM items (kv_split > 1): split s of an item visits key
  // tiles [s n_kt / kv_split, (s + 1) n_kt / kv_split) and writes its O / l in
  // float32 with its running max and sum; attn_merge_kernel combines the splits.
  int32_t kv_split;
  float* part_o;    // [kv_split][batch][n_q][n_heads * HD]
  float2* part_ml;  // [kv_split][batch][n_q][n_heads]: (running max, sum)
  int* status;
};

struct Work {
  int32_t b, h;
  bool is_ar;
  int64_t row0;     // first query row of tile 0
  int64_t seg_end;  // query rows >= seg_end are not in this segment
  int32_t n_kt;     // key tiles of the item (before any key split)
  int32_t split;    // key split of a DM item (0 when unsplit)
  int32_t kt0, kt1; // key tiles [kt0, kt1) this CTA visits
};

__device__ __forceinline__ Work decode_work(const Params& p) {
  Work w;
  int64_t bid = blockIdx.x;
  const int64_t items_dm = (int64_t)p.batch * p.n_heads * p.dm_pairs * p.kv_split;
  int32_t pairs;
  w.split = 0;
  if (bid < items_dm) {
    w.is_ar = false;
    pairs = p.dm_pairs;
    w.split = (int32_t)(bid % p.kv_split);
    bid /= p.kv_split;
  } else {
    bid -= items_dm;
    w.is_ar = true;
    pairs = p.ar_pairs;
  }
  w.b = (int32_t)(bid / ((int64_t)p.n_heads * pairs));
  const int64_t r = bid % ((int64_t)p.n_heads * pairs);
  w.h = (int32_t)(r / pairs);
  const int64_t pair = r % pairs;
  if (w.is_ar) {
    w.row0 = pair * 2 * BQ;
    w.seg_end = p.n_q_ar;
    const int64_t last = (w.row0 + 2 * BQ < w.seg_end ? w.row0 + 2 * BQ : w.seg_end) - 1;
    int64_t kmax = p.q_key_offset + last + 1;
    if (kmax > p.n_ar) kmax = p.n_ar;
    w.n_kt = (int32_t)((kmax + BKV - 1) / BKV);
  } else {
    w.row0 = p.n_q_ar + pair * 2 * BQ;
    w.seg_end = p.n_q;
    w.n_kt = (int32_t)((p.n_keys + BKV - 1) / BKV);
  }
  w.kt0 = (int32_t)((int64_t)w.split * w.n_kt / p.kv_split);
  w.kt1 = w.is_ar ? w.n_kt : (int32_t)((int64_t)(w.split + 1) * w.n_kt / p.kv_split);
  return w;
}

// Masking decisions of one query row, shared by the attention kernel and the
// debug export (cosmot_mot_mask_export), so that the export shows exactly what
// the kernel does.
struct RowMask {
  int64_t klimit;    // keys >= klimit are hidden (causal AR limit, or n_keys)
  int32_t my_chunk;  // block-causal DM rows: DM keys of later chunks are hidden
  bool bc_dm;
};

__device__ __forceinline__ RowMask row_mask(const Params& p, const Work& w, int64_t qi, bool valid) {
  RowMask m;
  const int64_t qk = p.q_key_offset + qi;  // key index of this query row
  m.bc_dm = !w.is_ar && p.mask_mode == COSMOT_MASK_BLOCK_CAUSAL;
  m.klimit = p.n_keys;
  if (w.is_ar) m.klimit = qk + 1 < p.n_ar ? qk + 1 : p.n_ar;
  // Rows past the segment are padding (never stored): they see everything,
  // so they never force the element-mask path on their warp.
  m.my_chunk = m.bc_dm ? (valid ? __ldg(p.chunk + qk) : INT32_MAX) : 0;
  return m;
}

// Chunk id of a key as the tile test sees it: AR keys and keys past the end
// never hide a tile (INT32_MIN).
__device__ __forceinline__ int32_t key_chunk_for_tile(const Params& p, int64_t key) {
  return (key >= p.n_ar && key < p.n_keys) ? __ldg(p.chunk + key) : INT32_MIN;
}

// A key tile needs per-element masks when it reaches past the row's key limit
// or (block-causal) holds a DM key of a later chunk; tile_chunk_max is the
// largest key_chunk_for_tile over its 128 keys.
__device__ __forceinline__ bool tile_needs_mask(const RowMask& m, int64_t kbase, int32_t tile_chunk_max) {
  return kbase + BKV > m.klimit || (m.bc_dm && tile_chunk_max > m.my_chunk);
}

__device__ __forceinline__ bool key_visible(const Params& p, const RowMask& m, int64_t key) {
  bool vis = key < m.klimit;
  if (m.bc_dm && key >= p.n_ar && vis) vis = __ldg(p.chunk + key) <= m.my_chunk;
  return vis;
}

// Key-tile skipping for block-causal DM work items.  A tile is visited iff
// its smallest key chunk is at most the largest chunk among the item's query
// rows (AR keys count as the smallest chunk, keys past the end are ignored):
// exactly the tiles that one of the item's rows sees.  FULL mode and AR items
// visit every tile of [0, n_kt).
__device__ __forceinline__ bool skips_tiles(const Params& p, const Work& w) { return p.skip && !w.is_ar; }

__device__ __forceinline__ int32_t key_chunk_for_visit(const Params& p, int64_t key) {
  if (key < p.n_ar) return INT32_MIN;
  return key < p.n_keys ? __ldg(p.chunk + key) : INT32_MAX;
}

// Largest chunk among the item's valid query rows (warp-cooperative).
__device__ __forceinline__ int32_t item_max_chunk(const Params& p, const Work& w, int lane) {
  int32_t m = INT32_MIN;
  for (int i = lane; i < 2 * BQ; i += 32) {
    const int64_t qi = w.row0 + i;
    if (qi < w.seg_end) m = max(m, __ldg(p.chunk + p.q_key_offset + qi));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
  return m;
}

// Smallest visited tile >= kt, or n_kt.
__device__ __forceinline__ int32_t next_visit(const uint32_t* visit, bool use, int32_t kt, int32_t n_kt) {
  if (!use) return kt < n_kt ? kt : n_kt;
  while (kt < n_kt) {
    const uint32_t word = visit[kt >> 5] >> (kt & 31);
    if (word) {
      kt += __ffs(word) - 1;
      return kt < n_kt ? kt : n_kt;
    }
    kt = (kt | 31) + 1;
  }
  return n_kt;
}

// kSkip: the instance that may skip block-causal DM tiles (p.skip set); the
// other one carries none of that machinery.
template <int HD, bool kSkip>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    mot_attention_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ Params p) {
  using C = Cfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sKV = sQ + 2 * C::TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (2 + SLOTS) * C::TILE_BYTES);
  const uint32_t bar_q = smem_u32(bars);
  const uint32_t bar_kv_full = bar_q + 8;                // [SLOTS]
  const uint32_t bar_kv_empty = bar_kv_full + 8 * SLOTS; // [SLOTS]
  const uint32_t bar_s_full = bar_kv_empty + 8 * SLOTS;  // [2]
  const uint32_t bar_p_half = bar_s_full + 16;           // [2] P of keys 0-63 written
  const uint32_t bar_p_full = bar_p_half + 16;           // [2] P of keys 64-127 written
  const uint32_t bar_o_done = bar_p_full + 16;           // [2]
  const uint32_t bar_drain = bar_o_done + 16;            // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1 + 2 * SLOTS + 9);
  uint32_t* visit = reinterpret_cast<uint32_t*>(smem + (2 + SLOTS) * C::TILE_BYTES + 256);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Work w = decode_work(p);
  const int32_t g = w.h / p.group;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < SLOTS; ++s) {
      mbar_init(bar_kv_full + 8 * s, 1);
      mbar_init(bar_kv_empty + 8 * s, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s_full + 8 * t, 1);
      mbar_init(bar_p_half + 8 * t, 4);  // one arrive per softmax warp
      mbar_init(bar_p_full + 8 * t, 4);
      mbar_init(bar_o_done + 8 * t, 1);
    }
    mbar_init(bar_drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  // Up to here the CTA touched only its own shared and tensor memory and the
  // kernel parameters, so this prologue may overlap the previous kernel.
  pdl_trigger();
  pdl_wait();
  bool use_visit = kSkip && skips_tiles(p, w);  // CTA-uniform
  if (use_visit) {
    // A tile is visited iff one of its keys is visible to the item's latest
    // chunk; each warp tests 32 consecutive keys (inside one tile) at a time
    // with coalesced loads and sets the tile's bit once if any passes.
    const int32_t n_words = (w.n_kt + 31) >> 5;
    for (int32_t i = threadIdx.x; i < n_words; i += NUM_THREADS) visit[i] = 0;
    const int32_t qmax = item_max_chunk(p, w, lane);
    __syncthreads();
    const int64_t span = (int64_t)w.n_kt * BKV;
    constexpr int U = 8;  // independent loads in flight per thread before any vote
    for (int64_t base = (int64_t)warp * 32; base < span; base += (int64_t)NUM_THREADS * U) {
      int32_t c[U];
#pragma unroll
      for (int u = 0; u < U; ++u) c[u] = key_chunk_for_visit(p, base + (int64_t)u * NUM_THREADS + lane);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t k0 = base + (int64_t)u * NUM_THREADS;  // 32 keys inside one tile
        if (__any_sync(0xffffffffu, c[u] <= qmax) && lane == 0 && k0 < span) {
          const int64_t kt = k0 / BKV;
          atomicOr(&visit[kt >> 5], 1u << (kt & 31));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  const int32_t n_kt = w.n_kt;
  const int32_t kt_begin = w.kt0, kt_end = w.kt1;  // this CTA's key tiles
  if (use_visit) {
    // Nothing to skip (a streaming block sees every cached key): walk the
    // tiles plainly.  Every thread reads the same words, so this stays uniform.
    bool all = true;
    for (int32_t wd = 0; wd < (n_kt >> 5); ++wd) all = all && visit[wd] == 0xffffffffu;
    if (n_kt & 31) all = all && (visit[n_kt >> 5] | (0xffffffffu << (n_kt & 31))) == 0xffffffffu;
    use_visit = !all;
  }

  if (warp < 4) {
  setmaxnreg_dec<kRegsIo>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      mbar_arrive_expect_tx(bar_q, 2 * C::TILE_BYTES);
      const int qrow = (int)(w.b * p.q_bstride + w.row0);
      for (int t = 0; t < 2; ++t)
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_2d(sQ + t * C::TILE_BYTES + bx * BOX_BYTES, &tmap_q, bar_q, w.h * HD + bx * 64, qrow + t * BQ);
      uint32_t armed_mask = 0, armed_parity = 0;
      const int kvrow = (int)(w.b * p.kv_bstride);
      // Load L = 2j (K) and 2j + 1 (V) of the j-th visited key tile.
      bool ok = true;
      for (int32_t kt = next_visit(visit, use_visit, kt_begin, kt_end), L = 0; kt < kt_end && ok;
           kt = next_visit(visit, use_visit, kt + 1, kt_end)) {
        for (int kv = 0; kv < 2; ++kv, ++L) {
          const int slot = L % SLOTS;
          const uint32_t par = (L / SLOTS) & 1;
          if (!mbar_wait(bar_kv_empty + 8 * slot, par ^ 1, p.status, kWhereAttnProducer)) {
            ok = false;
            break;
          }
          const uint32_t fb = bar_kv_full + 8 * slot;
          mbar_arrive_expect_tx(fb, C::TILE_BYTES);
          const CUtensorMap* m = kv ? &tmap_v : &tmap_k;
          const int krow = kvrow + kt * BKV;
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_2d(sKV + slot * C::TILE_BYTES + bx * BOX_BYTES, m, fb, g * HD + bx * 64, krow);
          armed_mask |= 1u << slot;
          armed_parity = (armed_parity & ~(1u << slot)) | (par << slot);
        }
      }
      // Let every bulk copy land before the CTA may exit.
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar_q, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
      }
      for (int s = 0; s < SLOTS; ++s)
        if (armed_mask & (1u << s)) {
          const uint32_t par = (armed_parity >> s) & 1u;
          const uint64_t t1 = globaltimer_ns();
          while (!mbar_try_wait(bar_kv_full + 8 * s, par) && globaltimer_ns() - t1 < kWaitLimitNs) {
          }
        }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      auto issue_s = [&](int t, int slot) {
        const uint32_t qa = sQ + t * C::TILE_BYTES;
        const uint32_t ka = sKV + slot * C::TILE_BYTES;
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t off = (k >> 2) * BOX_BYTES + (k & 3) * 32;
          umma_ss(tmem_base + C::s_col(t), sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024),
                  C::IDESC_S, k > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int slot, bool acc, int half) {  // keys 64*half .. 64*half+63
        const uint32_t va = sKV + slot * C::TILE_BYTES;
#pragma unroll
        for (int k = 4 * half; k < 4 * half + 4; ++k) {
          // V rows k*16 .. k*16+15: two 8-row swizzle atoms = 2048 bytes.
          umma_ts(tmem_base + C::o_col(t), tmem_base + C::s_col(t) + 8 * k, sw128_desc(va + 2048 * k, BOX_BYTES, 1024),
                  C::IDESC_O, (acc || k > 0) ? 1u : 0u);
        }
      };
      auto kv_wait = [&](int L) -> bool {
        return mbar_wait(bar_kv_full + 8 * (L % SLOTS), (L / SLOTS) & 1, p.status, kWhereAttnMma);
      };
      bool ok = mbar_wait(bar_q, 0, p.status, kWhereAttnMma) && kv_wait(0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        umma_commit(bar_s_full);
        issue_s(1, 0);
        umma_commit(bar_s_full + 8);
        umma_commit(bar_kv_empty + 8 * 0);
      }
      // j counts visited key tiles; kt is the j-th one.
      int32_t kt = next_visit(visit, use_visit, kt_begin, kt_end);
      for (int j = 0; kt < kt_end && ok; ++j) {
        const int32_t kt_next = next_visit(visit, use_visit, kt + 1, kt_end);
        const int LV = 2 * j + 1, LK = 2 * j + 2;
        const bool has_next = kt_next < kt_end;
        const uint32_t par = j & 1;
        // Order of the softmax events in steady state: tile 0 half, tile 0
        // full, tile 1 half, tile 1 full (tile 1 runs about half a block later).
        if (!kv_wait(LV) || !mbar_wait(bar_p_half, par, p.status, kWhereAttnMma)) break;
        tc_fence_after();
        issue_pv(0, LV % SLOTS, j > 0, 0);
        if (!mbar_wait(bar_p_full, par, p.status, kWhereAttnMma)) break;
        tc_fence_after();
        issue_pv(0, LV % SLOTS, true, 1);
        if (has_next) {
          if (!kv_wait(LK)) break;
          tc_fence_after();
          issue_s(0, LK % SLOTS);
          umma_commit(bar_s_full);
        }
        if (!mbar_wait(bar_p_half + 8, par, p.status, kWhereAttnMma)) break;
        tc_fence_after();
        issue_pv(1, LV % SLOTS, j > 0, 0);
        if (!mbar_wait(bar_p_full + 8, par, p.status, kWhereAttnMma)) break;
        tc_fence_after();
        issue_pv(1, LV % SLOTS, true, 1);
        umma_commit(bar_kv_empty + 8 * (LV % SLOTS));
        if (has_next) {
          issue_s(1, LK % SLOTS);
          umma_commit(bar_s_full + 8);
          umma_commit(bar_kv_empty + 8 * (LK % SLOTS));
        }
        kt = kt_next;
      }
      umma_commit(bar_o_done);
      umma_commit(bar_o_done + 8);
      umma_commit(bar_drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar_drain, 0)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          latch_status(p.status, COSMOT_ERR_TIMEOUT, kWhereAttnDrain);
          break;
        }
      }
    }
    __syncwarp();
  }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;           // query tile of this warpgroup
    const int lane_base = (warp & 3) * 32;   // TMEM lanes this warp may access
    const int r = lane_base + lane;
    const int64_t qi = w.row0 + (int64_t)t * BQ + r;
    const bool valid = qi < w.seg_end;
    const RowMask rm = row_mask(p, w, qi, valid);
    const uint32_t s_addr = tmem_base + ((uint32_t)lane_base << 16) + C::s_col(t);
    const uint32_t o_addr = tmem_base + ((uint32_t)lane_base << 16) + C::o_col(t);
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // j counts visited key tiles (it sets the barrier phases); kt is the j-th.
    int j = 0;
    for (int32_t kt = next_visit(visit, use_visit, kt_begin, kt_end); kt < kt_end;
         kt = next_visit(visit, use_visit, kt + 1, kt_end), ++j) {
      const int64_t kbase = (int64_t)kt * BKV;
      // Block-causal rows need element masks only where the tile holds a DM
      // key of a later chunk.  The warp reads the tile's 128 chunk ids (AR keys
      // and keys past the end count as visible) before waiting for S, so the
      // load latency hides behind the wait; the max is reduced after it.
      int32_t ck[4] = {INT32_MIN, INT32_MIN, INT32_MIN, INT32_MIN};
      if (rm.bc_dm) {
#pragma unroll
        for (int i = 0; i < 4; ++i) ck[i] = key_chunk_for_tile(p, kbase + lane + 32 * i);
      }
      // Warp-uniform decisions only: every tcgen05.ld/st below is .sync.aligned.
      if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full + 8 * t, j & 1, p.status, kWhereAttnSoftmax))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s[128];
      tmem_ld32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
      tmem_ld32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
      tmem_ld_wait();
      int32_t tmax = INT32_MIN;
      if (rm.bc_dm) {
        tmax = max(max(ck[0], ck[1]), max(ck[2], ck[3]));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) tmax = max(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
      }
      if (tile_needs_mask(rm, kbase, tmax)) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (!key_visible(p, rm, kbase + c)) s[c] = __float_as_uint(-INFINITY);
      }
      // Row max with four independent three-input chains (16 deep, not 128).
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 8) {
        mx0 = fmax3(mx0, __uint_as_float(s[c + 0]), __uint_as_float(s[c + 1]));
        mx1 = fmax3(mx1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
        mx2 = fmax3(mx2, __uint_as_float(s[c + 4]), __uint_as_float(s[c + 5]));
        mx3 = fmax3(mx3, __uint_as_float(s[c + 6]), __uint_as_float(s[c + 7]));
      }
      const float mt = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
      const float m_new = fmaxf(m, mt * sl2);
      const bool first = (m == -INFINITY);
      const bool need = !first && (m_new > m + kRescaleThreshold);
      float factor = 1.f;
      if (first) {
        m = m_new;
      } else if (need) {
        factor = ex2_approx(m - m_new);
        m = m_new;
        l *= factor;
      }
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(o_addr + 32 * c, ov);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * factor);
          tmem_st32(o_addr + 32 * c, ov);
        }
        tmem_st_wait();
      }
      const float mu = (m == -INFINITY) ? 0.f : m;
      float rs0 = 0.f, rs1 = 0.f;  // two running sums: half the dependent-add chain
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(s[c0 + 2 * e]), sl2, -mu));
          const float p1 = ex2_approx(fmaf(__uint_as_float(s[c0 + 2 * e + 1]), sl2, -mu));
          rs0 += p0;
          rs1 += p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st16(s_addr + (c0 >> 1), pk);
        if (c0 == 32) {  // P of keys 0-63 is in TMEM: PV over them may start
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_p_half + 8 * t);
        }
      }
      l += rs0 + rs1;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full + 8 * t);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(bar_o_done + 8 * t, 0, p.status, kWhereAttnSoftmax))) {
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      if (p.kv_split > 1 && !w.is_ar) {
        // one key split of the row: O / l in float32 with (running max, sum)
        const int64_t prow = ((int64_t)w.split * p.batch + w.b) * p.n_q + qi;
        float* pdst = p.part_o + prow * ((int64_t)p.n_heads * HD) + (int64_t)w.h * HD;
        const bool store = valid && dcheck(qi < p.n_q && w.split < p.kv_split, p.status, kWhereAttnStore);
        if (store) p.part_ml[prow * p.n_heads + w.h] = make_float2(m, l);
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(o_addr + 32 * c, ov);
          tmem_ld_wait();
          if (store) {
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              *reinterpret_cast<float4*>(pdst + 32 * c + 4 * q4) =
                  make_float4(__uint_as_float(ov[4 * q4]) * inv_l, __uint_as_float(ov[4 * q4 + 1]) * inv_l,
                              __uint_as_float(ov[4 * q4 + 2]) * inv_l, __uint_as_float(ov[4 * q4 + 3]) * inv_l);
          }
        }
      } else {
      __nv_bfloat16* dst = p.o + (w.b * p.o_bstride + qi) * p.ld_o + (int64_t)w.h * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32(o_addr + 32 * c, ov);
        tmem_ld_wait();
        if (valid && dcheck(qi < p.n_q && w.h < p.n_heads && w.b < p.batch, p.status, kWhereAttnStore)) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 v4;
            v4.x = pack_bf16x2(__uint_as_float(ov[8 * q4 + 0]) * inv_l, __uint_as_float(ov[8 * q4 + 1]) * inv_l);
            v4.y = pack_bf16x2(__uint_as_float(ov[8 * q4 + 2]) * inv_l, __uint_as_float(ov[8 * q4 + 3]) * inv_l);
            v4.z = pack_bf16x2(__uint_as_float(ov[8 * q4 + 4]) * inv_l, __uint_as_float(ov[8 * q4 + 5]) * inv_l);
            v4.w = pack_bf16x2(__uint_as_float(ov[8 * q4 + 6]) * inv_l, __uint_as_float(ov[8 * q4 + 7]) * inv_l);
            *reinterpret_cast<uint4*>(dst + 32 * c + 8 * q4) = v4;
          }
        }
      }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

template <int HD, bool kSkip>
cosmot_status launch(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const Params& p,
                     unsigned grid, cudaStream_t s) {
  static std::mutex mu;
  static uint64_t done_mask = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return COSMOT_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 64 || !(done_mask & (1ull << dev))) {
      if (cudaFuncSetAttribute(mot_attention_kernel<HD, kSkip>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg<HD>::SMEM_BYTES) != cudaSuccess)
        return COSMOT_ERR_CUDA;
      cudaFuncAttributes fa{};
      if (cudaFuncGetAttributes(&fa, mot_attention_kernel<HD, kSkip>) != cudaSuccess) return COSMOT_ERR_CUDA;
      // a build whose register count cannot fund the hand-over is not launched
      if (128 * kRegsIo + 256 * kRegsSoftmax > NUM_THREADS * fa.numRegs) return COSMOT_ERR_CUDA;
      if (dev < 64) done_mask |= 1ull << dev;
    }
  }
  return launch_status(launch_pdl(mot_attention_kernel<HD, kSkip>, dim3(grid), dim3(NUM_THREADS), Cfg<HD>::SMEM_BYTES,
                                  s, nullptr, tq, tk, tv, p));
}

}  // namespace attn
}  // namespace cosmot

namespace cosmot {
namespace attn {

// Descriptor checks and kernel parameters shared by the attention entry point
// and the mask export.
cosmot_status make_params(const cosmot_attn_desc* d, Params& p, int64_t& grid, int32_t kv_split = 1) {
  if (!d) return COSMOT_ERR_INVALID_ARG;
  const int hd = d->head_dim;
  if (hd != 64 && hd != 128) return COSMOT_ERR_UNSUPPORTED;
  if (d->n_heads < 1 || d->n_kv_heads < 1 || d->n_heads % d->n_kv_heads) return COSMOT_ERR_INVALID_ARG;
  if (d->n_q < 0 || d->n_keys < 1 || d->n_ar < 0 || d->n_ar > d->n_keys || d->q_key_offset < 0 ||
      d->q_key_offset + d->n_q > d->n_keys || d->batch < 1)
    return COSMOT_ERR_INVALID_ARG;
  if (d->mask_mode != COSMOT_MASK_FULL && d->mask_mode != COSMOT_MASK_BLOCK_CAUSAL) return COSMOT_ERR_INVALID_ARG;
  if (d->mask_mode == COSMOT_MASK_BLOCK_CAUSAL && !d->chunk) return COSMOT_ERR_INVALID_ARG;
  // the shared-memory visit mask of block-causal DM items holds kMaxVisitTiles key tiles
  if (d->mask_mode == COSMOT_MASK_BLOCK_CAUSAL && (d->n_keys + BKV - 1) / BKV > kMaxVisitTiles)
    return COSMOT_ERR_UNSUPPORTED;
  if (d->batch > 1 && (d->q_batch_stride < d->n_q || d->kv_batch_stride < d->n_keys || d->o_batch_stride < d->n_q))
    return COSMOT_ERR_INVALID_ARG;
  p = Params{};
  p.n_q = d->n_q;
  p.q_key_offset = d->q_key_offset;
  p.n_keys = d->n_keys;
  p.n_ar = d->n_ar;
  int64_t nqar = d->n_ar - d->q_key_offset;
  p.n_q_ar = nqar < 0 ? 0 : (nqar > d->n_q ? d->n_q : nqar);
  p.q_bstride = d->batch > 1 ? d->q_batch_stride : 0;
  p.kv_bstride = d->batch > 1 ? d->kv_batch_stride : 0;
  p.o_bstride = d->batch > 1 ? d->o_batch_stride : 0;
  p.n_heads = d->n_heads;
  p.group = d->n_heads / d->n_kv_heads;
  p.mask_mode = d->mask_mode;
  p.batch = d->batch;
  const int64_t ar_tiles = (p.n_q_ar + BQ - 1) / BQ;
  const int64_t dm_tiles = (p.n_q - p.n_q_ar + BQ - 1) / BQ;
  p.ar_pairs = (int32_t)((ar_tiles + 1) / 2);
  p.dm_pairs = (int32_t)((dm_tiles + 1) / 2);
  const float scale = d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / sqrtf((float)hd);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.chunk = d->chunk;
  p.skip = d->mask_mode == COSMOT_MASK_BLOCK_CAUSAL && !(d->flags & COSMOT_ATTN_NO_TILE_SKIP);
  p.status = device_status_ptr();
  if (!p.status) return COSMOT_ERR_CUDA;
  p.kv_split = kv_split;
  grid = (int64_t)d->batch * d->n_heads * (p.ar_pairs + (int64_t)p.dm_pairs * kv_split);
  if (grid > INT32_MAX) return COSMOT_ERR_UNSUPPORTED;
  return COSMOT_OK;
}

// One CTA per work item of the attention grid; only sequence 0, head 0 writes
// (the decisions depend on neither).  Thread i handles query row row0 + i.
__global__ void __launch_bounds__(2 * BQ) mask_export_kernel(const __grid_constant__ Params p, uint8_t* tile_codes,
                                                             int64_t n_kt_all, uint8_t* visible) {
  const Work w = decode_work(p);
  if (w.b != 0 || w.h != 0) return;
  const int64_t qi = w.row0 + threadIdx.x;
  if (qi >= w.seg_end) return;
  const RowMask rm = row_mask(p, w, qi, true);
  const bool skip = skips_tiles(p, w);
  int32_t qmax = INT32_MIN;  // the item's largest query chunk, as the kernel forms it
  if (skip)
    for (int i = 0; i < 2 * BQ; ++i)
      if (w.row0 + i < w.seg_end) qmax = max(qmax, __ldg(p.chunk + p.q_key_offset + w.row0 + i));
  for (int64_t j = 0; j < n_kt_all; ++j) {
    const int64_t kbase = j * BKV;
    uint8_t code = 0;
    bool masked = false;
    bool visited = j < w.n_kt;
    if (visited && skip) {
      int32_t mn = INT32_MAX;
      for (int c = 0; c < BKV; ++c) mn = min(mn, key_chunk_for_visit(p, kbase + c));
      visited = mn <= qmax;
    }
    if (visited) {
      int32_t tmax = INT32_MIN;
      if (rm.bc_dm)
        for (int c = 0; c < BKV; ++c) tmax = max(tmax, key_chunk_for_tile(p, kbase + c));
      masked = tile_needs_mask(rm, kbase, tmax);
      code = masked ? 2 : 1;
    }
    tile_codes[qi * n_kt_all + j] = code;
    if (visible)
      for (int c = 0; c < BKV && kbase + c < p.n_keys; ++c)
        visible[qi * p.n_keys + kbase + c] = (uint8_t)(code && (!masked || key_visible(p, rm, kbase + c)));
  }
}

}  // namespace attn
}  // namespace cosmot

namespace cosmot {
namespace attn {

// Combines the key splits of every (sequence, query row, head): with M the
// largest running max, weights w_s = l_s 2^(m_s - M) and O = sum_s w_s O_s /
// sum_s w_s, summed in split order (deterministic).  One warp per row and head,
// each lane HD/32 columns; a row no split saw (every w_s = 0) outputs 0.
template <int HD>
__global__ void __launch_bounds__(256) attn_merge_kernel(const Params p) {
  pdl_trigger();
  pdl_wait();
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t total = (int64_t)p.batch * (p.n_q - p.n_q_ar) * p.n_heads;
  if (warp >= total) return;
  const int32_t h = (int32_t)(warp % p.n_heads);
  const int64_t rb = warp / p.n_heads;              // (sequence, DM query row)
  const int32_t b = (int32_t)(rb / (p.n_q - p.n_q_ar));
  const int64_t qi = p.n_q_ar + rb % (p.n_q - p.n_q_ar);
  float mmax = -INFINITY;
  for (int s = 0; s < p.kv_split; ++s) {
    const float2 ml = p.part_ml[(((int64_t)s * p.batch + b) * p.n_q + qi) * p.n_heads + h];
    if (ml.y > 0.f) mmax = fmaxf(mmax, ml.x);
  }
  constexpr int C = HD / 32;
  float acc[C];
#pragma unroll
  for (int c = 0; c < C; ++c) acc[c] = 0.f;
  float wsum = 0.f;
  for (int s = 0; s < p.kv_split; ++s) {
    const int64_t prow = ((int64_t)s * p.batch + b) * p.n_q + qi;
    const float2 ml = p.part_ml[prow * p.n_heads + h];
    if (!(ml.y > 0.f)) continue;
    const float wgt = ml.y * ex2_approx(ml.x - mmax);
    wsum += wgt;
    const float* src = p.part_o + prow * ((int64_t)p.n_heads * HD) + (int64_t)h * HD + lane * C;
#pragma unroll
    for (int c = 0; c < C; ++c) acc[c] = fmaf(wgt, src[c], acc[c]);
  }
  const float inv = wsum > 0.f ? 1.0f / wsum : 0.f;
  if (!dcheck(qi < p.n_q && b < p.batch, p.status, kWhereAttnStore)) return;
  __nv_bfloat16* dst = p.o + (b * p.o_bstride + qi) * p.ld_o + (int64_t)h * HD + lane * C;
#pragma unroll
  for (int c = 0; c < C; c += 2) *reinterpret_cast<uint32_t*>(dst + c) = pack_bf16x2(acc[c] * inv, acc[c + 1] * inv);
}

// Bytes of the float32 partials of a key-split attention call.
size_t split_workspace_bytes(const cosmot_attn_desc* d, int32_t kv_split) {
  const int64_t rows = (int64_t)d->batch * d->n_q;
  return (size_t)kv_split * rows * d->n_heads * (size_t)d->head_dim * 4 + 256 +
         (size_t)kv_split * rows * d->n_heads * 8;
}

}  // namespace attn

int32_t attention_kv_split(int64_t dm_items, int64_t n_keys) {
  const int64_t n_kt = (n_keys + 127) / 128;
  const int64_t sms = num_sms();
  if (dm_items <= 0) return 1;
  auto eff = [&](int64_t s) {
    const int64_t u = dm_items * s;
    return (double)u / (double)(((u + sms - 1) / sms) * sms);
  };
  int32_t best = 1;
  for (int32_t s = 2; s <= 4 && s * 8 <= n_kt; ++s)
    if (eff(s) > eff(best) + 0.05) best = s;
  return best;
}

}  // namespace cosmot

extern "C" cosmot_status cosmot_attention_split_workspace(const cosmot_attn_desc* d, int32_t kv_split, size_t* bytes) {
  using namespace cosmot::attn;
  if (!d || !bytes || kv_split < 1 || kv_split > kMaxKvSplit || d->batch < 1 || d->n_q < 0 || d->n_heads < 1 ||
      (d->head_dim != 64 && d->head_dim != 128))
    return COSMOT_ERR_INVALID_ARG;
  *bytes = kv_split == 1 ? 0 : split_workspace_bytes(d, kv_split);
  return COSMOT_OK;
}

namespace cosmot {
namespace attn {

cosmot_status attention_impl(const cosmot_attn_desc* d, const void* q, int64_t ld_q, const void* k, const void* v,
                             int64_t ld_kv, void* o, int64_t ld_o, int32_t kv_split, void* workspace,
                             size_t workspace_bytes, cosmot_stream_t stream) {
  if (!d || !q || !k || !v || !o) return COSMOT_ERR_INVALID_ARG;
  if (kv_split < 1 || kv_split > kMaxKvSplit) return COSMOT_ERR_INVALID_ARG;
  Params p;
  int64_t grid = 0;
  cosmot_status st = make_params(d, p, grid, kv_split);
  if (st != COSMOT_OK) return st;
  const int hd = d->head_dim;
  const int64_t qcols = (int64_t)d->n_heads * hd, kvcols = (int64_t)d->n_kv_heads * hd;
  if (ld_q < qcols || ld_kv < kvcols || ld_o < qcols || ld_q % 8 || ld_kv % 8 || ld_o % 8) return COSMOT_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return COSMOT_ERR_INVALID_ARG;
  if (kv_split > 1) {
    // every split must visit at least one key tile: no tile skipping, and at
    // least kv_split key tiles
    if (p.skip) return COSMOT_ERR_UNSUPPORTED;
    if ((d->n_keys + BKV - 1) / BKV < kv_split) return COSMOT_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return COSMOT_ERR_INVALID_ARG;
    if (workspace_bytes < split_workspace_bytes(d, kv_split)) return COSMOT_ERR_WORKSPACE;
    const size_t o_bytes = ((size_t)kv_split * d->batch * d->n_q * d->n_heads * (size_t)hd * 4 + 255) & ~size_t(255);
    p.part_o = static_cast<float*>(workspace);
    p.part_ml = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + o_bytes);
  }
  if (d->n_q == 0) return COSMOT_OK;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.ld_o = ld_o;

  const int64_t q_rows = (d->batch - 1) * p.q_bstride + d->n_q;
  const int64_t kv_rows = (d->batch - 1) * p.kv_bstride + d->n_keys;
  if (q_rows + 2 * BQ > INT32_MAX || kv_rows + BKV > INT32_MAX) return COSMOT_ERR_UNSUPPORTED;

  CUtensorMap tq, tk, tv;
  st = make_tmap_bf16_2d(&tq, q, (uint64_t)q_rows, (uint64_t)qcols, (uint64_t)ld_q, BQ, 64);
  if (st != COSMOT_OK) return st;
  st = make_tmap_bf16_2d(&tk, k, (uint64_t)kv_rows, (uint64_t)kvcols, (uint64_t)ld_kv, BKV, 64);
  if (st != COSMOT_OK) return st;
  st = make_tmap_bf16_2d(&tv, v, (uint64_t)kv_rows, (uint64_t)kvcols, (uint64_t)ld_kv, BKV, 64);
  if (st != COSMOT_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (p.skip)
    return hd == 128 ? launch<128, true>(tq, tk, tv, p, (unsigned)grid, s)
                     : launch<64, true>(tq, tk, tv, p, (unsigned)grid, s);
  st = hd == 128 ? launch<128, false>(tq, tk, tv, p, (unsigned)grid, s)
                 : launch<64, false>(tq, tk, tv, p, (unsigned)grid, s);
  if (st != COSMOT_OK || kv_split == 1 || d->n_q == p.n_q_ar) return st;
  const int64_t warps = (int64_t)d->batch * (d->n_q - p.n_q_ar) * d->n_heads;
  const unsigned mgrid = (unsigned)((warps + 7) / 8);
  const cudaError_t e = hd == 128 ? launch_pdl(attn_merge_kernel<128>, dim3(mgrid), dim3(256), 0, s, nullptr, p)
                                  : launch_pdl(attn_merge_kernel<64>, dim3(mgrid), dim3(256), 0, s, nullptr, p);
  return launch_status(e);
}

}  // namespace attn
}  // namespace cosmot

extern "C" cosmot_status cosmot_mot_attention(const cosmot_attn_desc* d, const void* q, int64_t ld_q, const void* k,
                                              const void* v, int64_t ld_kv, void* o, int64_t ld_o,
                                              cosmot_stream_t stream) {
  return cosmot::attn::attention_impl(d, q, ld_q, k, v, ld_kv, o, ld_o, 1, nullptr, 0, stream);
}

extern "C" cosmot_status cosmot_mot_attention_split(const cosmot_attn_desc* d, const void* q, int64_t ld_q,
                                                    const void* k, const void* v, int64_t ld_kv, void* o,
                                                    int64_t ld_o, int32_t kv_split, void* workspace,
                                                    size_t workspace_bytes, cosmot_stream_t stream) {
  return cosmot::attn::attention_impl(d, q, ld_q, k, v, ld_kv, o, ld_o, kv_split, workspace, workspace_bytes,
                                      stream);
}

extern "C" int32_t cosmot_attention_kv_split(const cosmot_attn_desc* d) {
  if (!d || d->batch < 1 || d->n_heads < 1 || d->n_q < 0 || d->n_keys < 1) return 1;
  if (d->mask_mode == COSMOT_MASK_BLOCK_CAUSAL && !(d->flags & COSMOT_ATTN_NO_TILE_SKIP)) return 1;
  const int64_t nqar0 = d->n_ar - d->q_key_offset;
  const int64_t nqar = nqar0 < 0 ? 0 : (nqar0 > d->n_q ? d->n_q : nqar0);
  const int64_t dm_pairs = ((d->n_q - nqar + 127) / 128 + 1) / 2;
  return cosmot::attention_kv_split((int64_t)d->batch * d->n_heads * dm_pairs, d->n_keys);
}

extern "C" cosmot_status cosmot_mot_mask_export(const cosmot_attn_desc* d, uint8_t* tile_codes, uint8_t* visible,
                                                cosmot_stream_t stream) {
  using namespace cosmot;
  using namespace cosmot::attn;
  if (!tile_codes) return COSMOT_ERR_INVALID_ARG;
  Params p;
  int64_t grid = 0;
  cosmot_status st = make_params(d, p, grid);
  if (st != COSMOT_OK) return st;
  if (d->n_q == 0) return COSMOT_OK;
  const int64_t n_kt_all = (d->n_keys + BKV - 1) / BKV;
  mask_export_kernel<<<(unsigned)grid, 2 * BQ, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p, tile_codes, n_kt_all,
                                                                                             visible);
  return launch_status();
}
