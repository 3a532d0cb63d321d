// Block-sparse attention forward on sm_100a: tcgen05 tensor cores with TMEM
// accumulators, TMA-fed K/V ring indexed by per-q-tile kept lists.
//
// Sources: "Fast Video Generation with Sliding Tile Attention" explainer
// (aibr.jp/archives/60739), section 3 (attention restricted to kept tiles with a
// hardware-aware kernel); SPADE summary (gist.science/ja/paper/2608.03335),
// solution part 3 (head-wise sparse attention); NABLA explainer
// (aibr.jp/archives/124678), section 3 (block mask applied at block level).
// The arithmetic is softmax(Q K^T * scale + M) V with M = -inf outside kept
// block pairs, evaluated with an online (running max / running sum) softmax.
//
// Design (one persistent CTA per SM, 320 threads):
//   warps 0-3  softmax for q-tile slot 0 (thread = query row = TMEM lane)
//   warps 4-7  softmax for q-tile slot 1
//   warp  8    TMA producer: Q tiles, K/V tiles into an NSTAGE ring
//   warp  9    MMA issuer (one thread), also owns the TMEM allocation
// Units of two 128-row q-tiles are handed out dynamically: the producer warp takes
// the next unit index from a global counter (so all CTAs stay on a compact window
// of q-tiles, which keeps the K/V they read in L2, and the tail is balanced) and
// publishes it through a 4-entry shared-memory ring to the MMA and softmax warps.
// Each CTA processes a unit's two q-tiles (slots) in lock-step rounds;
// the MMA warp issues, per round r and slot s, O_s += P_s V_s,r then
// S_s = Q_s K_s,r+1^T, alternating slots, so that while one slot's softmax runs
// on the CUDA cores the tensor core works on the other slot.  TMEM (512 columns): S_0 | S_1 | O_0 | O_1, 128 columns
// each; P (bf16) is written over the first half of its slot's S columns and is
// the TMEM A operand of the P.V MMA.  The K/V ring stages are released by
// tcgen05.commit when the MMA that read them completes.
// Lazy rescaling: the running max used for the exponentials only moves when a
// row's new max exceeds it by more than 8 (log2 units), so O in TMEM is rarely
// touched by the softmax warps.
// Key tiles: with 128-token (or larger) key blocks a tile is 128 consecutive
// keys; with 64-token key blocks (template parameter kGather) a tile is any two
// kept key blocks of the list row, loaded as two 64-row TMA boxes into one tile.
// Paged K/V: the key rows of a tile come through a page table into a pool.
// All mbarrier waits are bounded; on expiry BSA_ERR_TIMEOUT is recorded in the
// workspace status word and every role leaves its loop.
#include <cudaTypedefs.h>

#include <mutex>

#include "bsa_common.cuh"
#include "tmem_io.cuh"
#include "attn_common.cuh"
#include "nvtx_range.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 320;
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
// The fast path keeps the running max while a tile's P sum stays <= 2^12.
constexpr float kFastSumLimit = 4096.0f;
// Optional software 2^x (FMA pipe) for BSA_POLY_PAIRS of every 16 column pairs of
// the fast path's exponentials, to relieve the MUFU (one exponential per 512 tensor
// FLOPs at head_dim 128); 0 by default: the FMA pipe's 128 lanes per SM clock
// spend about as many cycles on one polynomial exponential as the MUFU does (16
// per SM clock), and 2, 4 and 6 pairs in 16 measured 3-7 % slower on the radial
// and Sliding-Tile workloads.  BSA_POLY_EXP2=1 is the older spelling of 4 in 16.
#ifndef BSA_POLY_EXP2
#define BSA_POLY_EXP2 0
#endif
#ifndef BSA_POLY_PAIRS
#define BSA_POLY_PAIRS (BSA_POLY_EXP2 ? 4 : 0)
#endif
constexpr int kPolyPairs = BSA_POLY_PAIRS;
static_assert(kPolyPairs >= 0 && kPolyPairs <= 16, "BSA_POLY_PAIRS is 0..16");
// Pair i of a 16-pair chunk goes to the polynomial: spread evenly over the chunk.
__device__ __forceinline__ constexpr bool poly_pair(int i) {
  return kPolyPairs > 0 && (i * kPolyPairs) % 16 < kPolyPairs;
}
// Lazy-rescale threshold in log2 units (the running max in use may trail the true
// one by up to this much, so fast-path P values stay below 2^threshold).
#ifndef BSA_RESCALE_THRESHOLD
#define BSA_RESCALE_THRESHOLD 8.0f
#endif
constexpr float kRescaleThreshold = BSA_RESCALE_THRESHOLD;  // log2 units

// Optional phase timestamps (SM clock) of CTA 0 for latency analysis; compiled
// only with -DBSA_TRACE and read back with bsa_trace_dump().
#ifdef BSA_TRACE
__device__ unsigned long long g_bsa_trace[1 << 16];
#define BSA_TRACE_AT(idx) \
  do {                    \
    if (blockIdx.x == 0 && (idx) < (1 << 16)) g_bsa_trace[(idx)] = clock64(); \
  } while (0)
#else
#define BSA_TRACE_AT(idx) \
  do {                    \
  } while (0)
#endif

template <int D>
struct Cfg {
  static constexpr int KCH = D / 64;                  // 128-byte swizzle chunks per row
  static constexpr int CHUNK_BYTES = kBM * 128;       // one chunk of a 128-row tile
  static constexpr int TILE_BYTES = KCH * CHUNK_BYTES;
  static constexpr int NSTAGE = D == 128 ? 5 : 10;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = 2 * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_RING + NSTAGE * TILE_BYTES;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
};

struct AttnParams {
  int B, H, nq, nk, QT;
  int block_q, block_k, QB, LR, list_heads, expand;
  int total_items, total_units;
  float scale_log2;
  const int* row_ptr;
  const int* cnt;
  const uint32_t* entries;
  __nv_bfloat16* o;
  long long o_stride;  // elements between consecutive token rows of o
  float* lse;
  int* status;
  int* unit_counter;  // next unit to hand out (zeroed before the launch)
  unsigned long long timeout_ns;
  // paged K/V: logical 128-key tile kt of batch b is physical page
  // page_table[b * pages_per_batch + kt] of a one-batch pool (nullptr: contiguous)
  const int* page_table;
  int pages_per_batch;
  // 64-token key blocks: list entries name two arbitrary key blocks per tile
  // (block, block + 1 or 0, quadrant bits) instead of one 128-key tile
  int gather_k;
};

// Key row (in the K/V tensor or pool) of 64-token key block kb of batch b.
__device__ __forceinline__ int key_block_row(const AttnParams& p, int b, int kb) {
  if (p.page_table)
    return __ldg(p.page_table + static_cast<long long>(b) * p.pages_per_batch + (kb >> 1)) * kBN +
           (kb & 1) * 64;
  return kb * 64;
}

struct Item {
  int b, h, qt, n;  // n < 0: no item; n == 0: empty kept list
  const uint32_t* ent;
};

__device__ __forceinline__ Item get_item(const AttnParams& p, int it) {
  Item r;
  r.n = -1;
  r.ent = nullptr;
  r.b = r.h = r.qt = 0;
  if (it >= p.total_items) return r;
  r.qt = it % p.QT;
  const int bh = it / p.QT;
  r.h = bh % p.H;
  r.b = bh / p.H;
  const int mh = p.list_heads == 1 ? 0 : bh;
  const int lr = p.block_q >= 128 ? (r.qt * kBM) / p.block_q : r.qt;
  const int first_qb = p.block_q >= 128 ? lr : 2 * lr;
  r.n = p.cnt[mh * p.LR + lr];
  r.ent = p.entries + static_cast<long long>(p.row_ptr[mh * p.QB + first_qb]) * p.expand;
  return r;
}

// Both slots of a unit read the same K/V stream: same batch, head and kept list.
__device__ __forceinline__ bool shares_kv(const Item& a, const Item& b) {
  return a.n > 0 && b.n == a.n && a.ent == b.ent && a.b == b.b && a.h == b.h;
}

// ---------------------------------------------------------------------------
// The attention kernel.
// ---------------------------------------------------------------------------
template <int D, bool kGather>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmK64,
                    const __grid_constant__ CUtensorMap tmV64, const AttnParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sRing = sbase + C::OFF_RING;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  // barrier slots
  const uint32_t bar0 = smem_u32(bars);
  auto FULL = [&](int i) { return bar0 + 8u * i; };
  auto EMPTY = [&](int i) { return bar0 + 8u * (C::NSTAGE + i); };
  auto QFULL = [&](int s) { return bar0 + 8u * (2 * C::NSTAGE + s); };
  auto QEMPTY = [&](int s) { return bar0 + 8u * (2 * C::NSTAGE + 2 + s); };
  auto SFULL = [&](int s) { return bar0 + 8u * (2 * C::NSTAGE + 4 + s); };
  auto PREADY = [&](int s) { return bar0 + 8u * (2 * C::NSTAGE + 6 + s); };
  auto ODONE = [&](int s) { return bar0 + 8u * (2 * C::NSTAGE + 8 + s); };
  const uint32_t FINAL = bar0 + 8u * (2 * C::NSTAGE + 10);
  // unit hand-off ring: the producer takes units from the global counter and
  // publishes them to the MMA thread and the softmax warps
  auto UFULL = [&](int i) { return bar0 + 8u * (2 * C::NSTAGE + 11 + i); };
  auto UEMPTY = [&](int i) { return bar0 + 8u * (2 * C::NSTAGE + 15 + i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 8 * (2 * C::NSTAGE + 19));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(tmem_slot + 2);
  constexpr int kUnitConsumers = 1 + 8;  // MMA thread + one arrival per softmax warp

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(FULL(i), 1);
      mbar_init(EMPTY(i), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(QFULL(s), 1);
      mbar_init(QEMPTY(s), 1);
      mbar_init(SFULL(s), 1);
      mbar_init(PREADY(s), 4);
      mbar_init(ODONE(s), 1);
    }
    mbar_init(FINAL, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(UFULL(i), 1);
      mbar_init(UEMPTY(i), kUnitConsumers);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == kLoadWarp && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 8) {
  // third warpgroup (two warps): producer and MMA issuer
  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ producer
    // Ring order (must match the MMA issuer): per unit, K of step 0 for each slot,
    // then per round r and slot s: V(s, r) followed by K(s, r + 1).
    if (lane == 0) {
      int st = 0;
      uint32_t ph = 0;
      uint32_t qph[2] = {0, 0};
      uint32_t filled = 0, fill_phase = 0;  // per stage: ever filled / phase of the last fill
      int q_filled[2] = {-1, -1};
      bool ok = true;
      int gld = 0;
      (void)gld;
      auto load_tile = [&](const CUtensorMap* map, const CUtensorMap* map64, const Item& itm,
                           int step) -> bool {
        const int tix = 32768 + min(gld++, 8191) * 2;
        BSA_TRACE_AT(tix + 0);
        if (!mbar_wait(EMPTY(st), ph ^ 1u, abort_flag, p.status, p.timeout_ns)) return false;
        BSA_TRACE_AT(tix + 1);
        const uint32_t ent = __ldg(itm.ent + step);
        const int bco = p.page_table ? 0 : itm.b;
        mbar_expect_tx(FULL(st), C::TILE_BYTES);
        if constexpr (kGather) {
          // two 64-row boxes; a missing second block repeats the first (its columns
          // are masked, the rows only need to be finite)
          const int kb0 = static_cast<int>(ent & 0x3FFFu);
          const int kb1p = static_cast<int>((ent >> 14) & 0x3FFFu);
          const int r0 = key_block_row(p, itm.b, kb0);
          const int r1 = key_block_row(p, itm.b, kb1p ? kb1p - 1 : kb0);
#pragma unroll
          for (int c = 0; c < C::KCH; ++c) {
            const uint32_t dst = sRing + st * C::TILE_BYTES + c * C::CHUNK_BYTES;
            tma_load_4d(dst, map64, FULL(st), 64 * c, itm.h, r0, bco);
            tma_load_4d(dst + C::CHUNK_BYTES / 2, map64, FULL(st), 64 * c, itm.h, r1, bco);
          }
        } else {
          const int kt = static_cast<int>(ent & 0x0FFFFFFFu);
          const int row = p.page_table
                              ? __ldg(p.page_table + static_cast<long long>(itm.b) * p.pages_per_batch + kt) * kBN
                              : kt * kBN;
#pragma unroll
          for (int c = 0; c < C::KCH; ++c)
            tma_load_4d(sRing + st * C::TILE_BYTES + c * C::CHUNK_BYTES, map, FULL(st), 64 * c,
                        itm.h, row, bco);
        }
        filled |= 1u << st;
        fill_phase = (fill_phase & ~(1u << st)) | (ph << st);
        if (++st == C::NSTAGE) { st = 0; ph ^= 1u; }
        return true;
      };
      for (int uk = 0; ok; ++uk) {
        // take the next unit and publish it to the other roles
        const int slot = uk & 3;
        if (!mbar_wait(UEMPTY(slot), ((uk >> 2) & 1) ^ 1u, abort_flag, p.status, p.timeout_ns)) {
          ok = false;
          break;
        }
        const int u = atomicAdd(p.unit_counter, 1);
        unit_ring[slot] = u;
        mbar_arrive(UFULL(slot));
        if (u >= p.total_units) break;
        Item it[2] = {get_item(p, 2 * u), get_item(p, 2 * u + 1)};
        for (int s = 0; s < 2 && ok; ++s) {
          if (it[s].n <= 0) continue;
          ok = mbar_wait(QEMPTY(s), qph[s] ^ 1u, abort_flag, p.status, p.timeout_ns);
          if (!ok) break;
          q_filled[s] = static_cast<int>(qph[s]);
          qph[s] ^= 1u;
          mbar_expect_tx(QFULL(s), C::TILE_BYTES);
          for (int c = 0; c < C::KCH; ++c)
            tma_load_4d(sQ + s * C::TILE_BYTES + c * C::CHUNK_BYTES, &tmQ, QFULL(s), 64 * c,
                        it[s].h, it[s].qt * kBM, it[s].b);
        }
        if (shares_kv(it[0], it[1])) {  // one K/V stream read by both slots
          const int n = it[0].n;
          ok = ok && load_tile(&tmK, &tmK64, it[0], 0);
          for (int r = 0; r < n && ok; ++r) {
            ok = load_tile(&tmV, &tmV64, it[0], r);
            if (ok && r + 1 < n) ok = load_tile(&tmK, &tmK64, it[0], r + 1);
          }
          continue;
        }
        for (int s = 0; s < 2 && ok; ++s)
          if (it[s].n > 0) ok = load_tile(&tmK, &tmK64, it[s], 0);
        const int R = max(it[0].n, it[1].n);
        for (int r = 0; r < R && ok; ++r) {
          for (int s = 0; s < 2 && ok; ++s) {
            if (r >= it[s].n) continue;
            ok = load_tile(&tmV, &tmV64, it[s], r);
            if (ok && r + 1 < it[s].n) ok = load_tile(&tmK, &tmK64, it[s], r + 1);
          }
        }
      }
      // Do not leave the CTA while a TMA copy into its shared memory may be in flight.
      for (int i = 0; i < C::NSTAGE; ++i)
        if (filled & (1u << i))
          mbar_wait_drain(FULL(i), (fill_phase >> i) & 1u, p.status, p.timeout_ns);
      for (int s = 0; s < 2; ++s)
        if (q_filled[s] >= 0)
          mbar_wait_drain(QFULL(s), static_cast<uint32_t>(q_filled[s]), p.status, p.timeout_ns);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // Per slot the tensor core alternates P.V of step r and Q.K^T of step r + 1, the
    // two slots interleaved: while slot A's softmax runs, slot B's P.V and next
    // Q.K^T execute, and the reverse.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, 0, 1);
      int st = 0;
      uint32_t ph = 0;
      uint32_t qph[2] = {0, 0}, pph[2] = {0, 0};
      bool ok = true;
      int gop = 0;
      (void)gop;
      // Descriptors are built once; per MMA only the 14-bit start-address field
      // (16-byte units, shared memory < 256 KB so no carry) moves by a constant.
      const uint64_t dq0 = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(sRing, 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(sRing, C::CHUNK_BYTES, 1024);
      constexpr uint32_t kTileUnits = C::TILE_BYTES >> 4;
      // Wait for the next ring stage in fill order and return its index.
      auto acquire = [&](int& stage) -> bool {
        const int tix = 16384 + min(gop++, 4095) * 4;
        BSA_TRACE_AT(tix + 0);
        if (!mbar_wait(FULL(st), ph, abort_flag, p.status, p.timeout_ns)) return false;
        BSA_TRACE_AT(tix + 1);
        stage = st;
        if (++st == C::NSTAGE) { st = 0; ph ^= 1u; }
        return true;
      };
      // S_s = Q_s K^T, K in ring stage `stage`.
      auto qk = [&](int s, int stage) {
        tc_fence_after();
        const uint64_t da = dq0 + static_cast<uint64_t>(s * kTileUnits);
        const uint64_t db = dk0 + static_cast<uint64_t>(stage * kTileUnits);
        const uint32_t dt = tmem + s * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off =
              static_cast<uint64_t>((((kk >> 2) * C::CHUNK_BYTES) + (kk & 3) * 32) >> 4);
          mma_ss(dt, da + off, db + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // O_s (+)= P_s V once slot s's softmax has published P.
      auto pv = [&](int s, int stage, int step) -> bool {
        if (!mbar_wait(PREADY(s), pph[s], abort_flag, p.status, p.timeout_ns)) return false;
        tc_fence_after();
        const uint64_t db = dv0 + static_cast<uint64_t>(stage * kTileUnits);
        const uint32_t dt = tmem + 256 + s * 128;
        const uint32_t ta = tmem + s * 128;
        const uint32_t acc0 = step > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts(dt, ta + kk * 8, db + static_cast<uint64_t>(kk * (16 * 128 / 16)), idesc_pv,
                 kk > 0 ? 1u : acc0);
        pph[s] ^= 1u;
        return true;
      };
      for (int uk = 0; ok; ++uk) {
        const int slot = uk & 3;
        if (!mbar_wait(UFULL(slot), (uk >> 2) & 1, abort_flag, p.status, p.timeout_ns)) {
          ok = false;
          break;
        }
        const int u = unit_ring[slot];
        mbar_arrive(UEMPTY(slot));
        if (u >= p.total_units) break;
        Item it[2] = {get_item(p, 2 * u), get_item(p, 2 * u + 1)};
        if (shares_kv(it[0], it[1])) {
          const int n = it[0].n;
          int ks = 0, vs = 0;
          for (int s = 0; s < 2 && ok; ++s) {
            ok = mbar_wait(QFULL(s), qph[s], abort_flag, p.status, p.timeout_ns);
            qph[s] ^= 1u;
          }
          if (!ok || !acquire(ks)) { ok = false; break; }
          qk(0, ks);
          mma_commit(SFULL(0));
          qk(1, ks);
          mma_commit(EMPTY(ks));
          mma_commit(SFULL(1));
          if (n == 1) { mma_commit(QEMPTY(0)); mma_commit(QEMPTY(1)); }
          for (int r = 0; r < n && ok; ++r) {
            const bool more = r + 1 < n;
            if (!acquire(vs) || !pv(0, vs, r)) { ok = false; break; }
            if (r == n - 1) mma_commit(ODONE(0));
            if (more) {
              if (!acquire(ks)) { ok = false; break; }
              qk(0, ks);
              mma_commit(SFULL(0));
              if (r + 1 == n - 1) mma_commit(QEMPTY(0));
            }
            if (!pv(1, vs, r)) { ok = false; break; }
            mma_commit(EMPTY(vs));
            if (r == n - 1) mma_commit(ODONE(1));
            if (more) {
              qk(1, ks);
              mma_commit(EMPTY(ks));
              mma_commit(SFULL(1));
              if (r + 1 == n - 1) mma_commit(QEMPTY(1));
            }
          }
          continue;
        }
        for (int s = 0; s < 2 && ok; ++s) {
          if (it[s].n <= 0) continue;
          int ks = 0;
          ok = mbar_wait(QFULL(s), qph[s], abort_flag, p.status, p.timeout_ns) && acquire(ks);
          if (!ok) break;
          qph[s] ^= 1u;
          qk(s, ks);
          mma_commit(EMPTY(ks));
          mma_commit(SFULL(s));
          if (it[s].n == 1) mma_commit(QEMPTY(s));
        }
        const int R = max(it[0].n, it[1].n);
        for (int r = 0; r < R && ok; ++r) {
          for (int s = 0; s < 2 && ok; ++s) {
            const int n = it[s].n;
            if (r >= n) continue;
            int vs = 0, ks = 0;
            if (!acquire(vs) || !pv(s, vs, r)) { ok = false; break; }
            mma_commit(EMPTY(vs));
            if (r == n - 1) mma_commit(ODONE(s));
            if (r + 1 < n) {
              if (!acquire(ks)) { ok = false; break; }
              qk(s, ks);
              mma_commit(EMPTY(ks));
              mma_commit(SFULL(s));
              if (r + 1 == n - 1) mma_commit(QEMPTY(s));
            }
          }
        }
      }
      // Every MMA of this CTA has finished before TMEM is released.
      mma_commit(FINAL);
      mbar_wait_drain(FINAL, 0, p.status, p.timeout_ns);
    }
  }
  } else {
    // ------------------------------------------------------------ softmax (8 warps)
    const int s = warp >> 2;                 // slot
    const int row = threadIdx.x & 127;       // query row within the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + s * 128;
    const uint32_t tO = tmem + lane_base + 256 + s * 128;
    const float sl2 = p.scale_log2;
    uint32_t sph = 0, oph = 0;
    int gstep = 0;
    (void)gstep;
    bool ok = true;
    for (int uk = 0; ok; ++uk) {
      const int slot = uk & 3;
      if (!mbar_wait(UFULL(slot), (uk >> 2) & 1, abort_flag, p.status, p.timeout_ns)) {
        ok = false;
        break;
      }
      const int u = unit_ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(UEMPTY(slot));
      if (u >= p.total_units) break;
      const Item me = get_item(p, 2 * u + s);
      if (me.n < 0) continue;
      const int qrow = me.qt * kBM + row;
      float m_used = -INFINITY, l = 0.f;
      const int qh = row >> 6;
      uint32_t ent_next = me.n > 0 ? __ldg(me.ent) : 0u;
      for (int j = 0; j < me.n; ++j) {
        const uint32_t ent = ent_next;
        if (j + 1 < me.n) ent_next = __ldg(me.ent + j + 1);
        const int tix = (warp & 3) == 0 && lane == 0 ? s * 8192 + min(gstep, 1023) * 8 : (1 << 16);
        BSA_TRACE_AT(tix + 0);
        ok = mbar_wait(SFULL(s), sph, abort_flag, p.status, p.timeout_ns);
        BSA_TRACE_AT(tix + 1);
        ++gstep;
        if (!ok) break;
        sph ^= 1u;
        tc_fence_after();
        const uint32_t bits = ent >> 28;
        // keys that exist: in the tile (adjacent blocks) or in each 64-column half
        // (gathered blocks)
        int kvalid = 0, v0 = 64, v1 = 64;
        if constexpr (kGather) {
          const int kb0 = static_cast<int>(ent & 0x3FFFu);
          const int kb1p = static_cast<int>((ent >> 14) & 0x3FFFu);
          v0 = min(64, p.nk - kb0 * 64);
          v1 = kb1p ? min(64, p.nk - (kb1p - 1) * 64) : 64;  // an empty half is masked by bits
        } else {
          kvalid = p.nk - static_cast<int>(ent & 0x0FFFFFFFu) * kBN;
        }
        const bool ragged = kGather ? (v0 < 64 || v1 < 64) : kvalid < kBN;
        // Quadrant mask of 64-token blocks: each warp's 32 rows lie in one q-half, so
        // whether a 64-column half is kept is uniform across the warp.
        const bool lo_ok = (bits >> (qh * 2)) & 1u, hi_ok = (bits >> (qh * 2 + 1)) & 1u;
        float lsum = 0.f;
        bool done = false;
        // Fast path (every tile after the first, running max finite, no ragged tail):
        // one pass over S against the running max, the next 32 columns loading while
        // the current ones are exponentiated; P stays in registers until the tile's
        // P sum is known to be <= kFastSumLimit, which bounds every P (an overflow
        // to inf fails the test too).  Otherwise the general path below redoes the
        // tile from S, which is still intact in TMEM.
        if (j > 0 && !ragged && __all_sync(0xffffffffu, m_used != -INFINITY)) {
          uint32_t pk[64];
          float2 lpa = make_float2(0.f, 0.f), lpb = make_float2(0.f, 0.f);
          const float2 sl2x2 = make_float2(sl2, sl2);
          const float2 negm = make_float2(-m_used, -m_used);
          uint32_t ra[32], rb[32];
          auto exp_chunk = [&](const uint32_t* cur, uint32_t* out) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 x = ffma2(make_float2(__uint_as_float(cur[2 * i]),
                                                 __uint_as_float(cur[2 * i + 1])),
                                     sl2x2, negm);
              float2 pp;
              if (poly_pair(i)) {
                pp = poly_exp2x2(x);
              } else {
                pp.x = fast_exp2(x.x);
                pp.y = fast_exp2(x.y);
              }
              if (i & 1) lpb = fadd2(lpb, pp); else lpa = fadd2(lpa, pp);
              __nv_bfloat162 h2 = __floats2bfloat162_rn(pp.x, pp.y);
              out[i] = *reinterpret_cast<uint32_t*>(&h2);
            }
          };
          if (lo_ok && hi_ok) {
            // Whole tile kept (every Sliding-Tile / radial step): no per-chunk tests.
            tmem_ld32x32b_x32_nowait(tS, ra);
            tmem_wait_ld_x32(ra);
            tmem_ld32x32b_x32_nowait(tS + 32, rb);
            exp_chunk(ra, pk);
            tmem_wait_ld_x32(rb);
            tmem_ld32x32b_x32_nowait(tS + 64, ra);
            exp_chunk(rb, pk + 16);
            tmem_wait_ld_x32(ra);
            tmem_ld32x32b_x32_nowait(tS + 96, rb);
            exp_chunk(ra, pk + 32);
            tmem_wait_ld_x32(rb);
            exp_chunk(rb, pk + 48);
          } else {
            if (lo_ok) {
              tmem_ld32x32b_x32_nowait(tS, ra);
              tmem_wait_ld_x32(ra);
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const bool cur_ok = c < 2 ? lo_ok : hi_ok;
              const bool nxt_ok = c + 1 < 2 ? lo_ok : hi_ok;
              uint32_t* cur = (c & 1) ? rb : ra;
              uint32_t* nxt = (c & 1) ? ra : rb;
              if (c < 3 && nxt_ok) tmem_ld32x32b_x32_nowait(tS + (c + 1) * 32, nxt);
              if (cur_ok) {
                exp_chunk(cur, pk + c * 16);
              } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[c * 16 + i] = 0u;
              }
              if (c < 3 && nxt_ok) tmem_wait_ld_x32(nxt);
            }
          }
          BSA_TRACE_AT(tix + 5);
          const float tile_sum = (lpa.x + lpa.y) + (lpb.x + lpb.y);
          if (__all_sync(0xffffffffu, tile_sum <= kFastSumLimit)) {
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_st32x32b_x16(tS + c * 16, pk + c * 16);
            BSA_TRACE_AT(tix + 6);
            lsum = tile_sum;
            done = true;
          }
        }
        float alpha = 1.0f;
        bool rescale_o = false;
        if (!done) {
          // General path: pass 1 takes the tile's row max, then the running max is
          // moved lazily (only when it grew by more than the threshold; O in TMEM and
          // l are then scaled by alpha -- O holds data only once a finite base has
          // been used), pass 2 writes P.  Handles the first tile, masked quadrants,
          // the ragged key tail and rows whose max jumped.
          float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c0 = 0; c0 < kBN; c0 += 64) {
            const bool half_ok = c0 < 64 ? lo_ok : hi_ok;
            if (!half_ok) continue;
            uint32_t sr[64];
            tmem_ld32x32b_x64(tS + c0, sr);
            if (!ragged) {
#pragma unroll
              for (int i = 0; i < 64; ++i) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(sr[i]));
            } else {
#pragma unroll
              for (int i = 0; i < 64; ++i)
                if (kGather ? i < (c0 < 64 ? v0 : v1) : c0 + i < kvalid)
                  mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(sr[i]));
            }
          }
          const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
          const float m_new = fmaxf(m_used, mt);
          if (j == 0) {
            m_used = m_new;
          } else if (m_new > m_used + kRescaleThreshold) {
            if (m_used != -INFINITY) {
              alpha = fast_exp2(m_used - m_new);
              rescale_o = true;
            }
            m_used = m_new;
          }
          const float msub = m_used == -INFINITY ? 0.f : m_used;
          float lp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c0 = 0; c0 < kBN; c0 += 32) {
            const bool half_ok = c0 < 64 ? lo_ok : hi_ok;
            uint32_t pk[16];
            if (!half_ok) {
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[i] = 0u;
            } else {
              uint32_t sr[32];
              tmem_ld32x32b_x32(tS + c0, sr);
              if (!ragged) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const float p0 = fast_exp2(fmaf(__uint_as_float(sr[2 * i]), sl2, -msub));
                  const float p1 = fast_exp2(fmaf(__uint_as_float(sr[2 * i + 1]), sl2, -msub));
                  lp[(2 * i) & 3] += p0;
                  lp[(2 * i + 1) & 3] += p1;
                  __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                  pk[i] = *reinterpret_cast<uint32_t*>(&h2);
                }
              } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  // gathered: column within its half against that half's keys
                  const int c = kGather ? (c0 & 63) + 2 * i : c0 + 2 * i;
                  const int hv = kGather ? (c0 < 64 ? v0 : v1) : kvalid;
                  const float p0 =
                      c < hv ? fast_exp2(fmaf(__uint_as_float(sr[2 * i]), sl2, -msub)) : 0.f;
                  const float p1 = c + 1 < hv
                                       ? fast_exp2(fmaf(__uint_as_float(sr[2 * i + 1]), sl2, -msub))
                                       : 0.f;
                  lp[(2 * i) & 3] += p0;
                  lp[(2 * i + 1) & 3] += p1;
                  __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                  pk[i] = *reinterpret_cast<uint32_t*>(&h2);
                }
              }
            }
            tmem_st32x32b_x16(tS + c0 / 2, pk);
          }
          lsum = (lp[0] + lp[1]) + (lp[2] + lp[3]);
        }
        if (__any_sync(0xffffffffu, rescale_o)) {  // rare: O is idle until P is signalled
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 16) {
            uint32_t ov[16];
            tmem_ld32x32b_x16(tO + c0, ov);
#pragma unroll
            for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st32x32b_x16(tO + c0, ov);
          }
        }
        l = fmaf(l, alpha, lsum);
        BSA_TRACE_AT(tix + 2);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(PREADY(s));
        BSA_TRACE_AT(tix + 3);
      }
      if (!ok) break;
      __nv_bfloat16* orow =
          p.o + (static_cast<long long>(me.b) * p.nq + qrow) * p.o_stride + static_cast<long long>(me.h) * D;
      float* lrow = p.lse + (static_cast<long long>(me.b) * p.H + me.h) * p.nq + qrow;
      if (me.n == 0) {
        if (qrow < p.nq) {
          uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(orow)[c] = z;
          *lrow = -INFINITY;
        }
        continue;
      }
      ok = mbar_wait(ODONE(s), oph, abort_flag, p.status, p.timeout_ns);
      if (!ok) break;
      oph ^= 1u;
      tc_fence_after();
      const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t ov[32];
        tmem_ld32x32b_x32(tO + c0, ov);
        if (qrow < p.nq) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(ov[2 * i]) * inv,
                                                      __uint_as_float(ov[2 * i + 1]) * inv);
            pk[i] = *reinterpret_cast<uint32_t*>(&h2);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          dst[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
          dst[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
        }
      }
      if (qrow < p.nq) *lrow = l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      // O is read out; the next item's first P.V may overwrite it once P is ready
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int D>
int launch_attn(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                const CUtensorMap& mk64, const CUtensorMap& mv64,
                const AttnParams& p, cudaStream_t st) {
  using C = Cfg<D>;
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_fwd_kernel<D, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return record_cuda_error(e);
    if (dev >= 0 && dev < 64) attr_done[dev] = true;
  }
  int grid = device_sm_count();
  if (grid > p.total_units) grid = p.total_units;
  if (p.gather_k)
    attn_fwd_kernel<D, true><<<grid, kThreads, C::SMEM, st>>>(mq, mk, mv, mk64, mv64, p);
  else
    attn_fwd_kernel<D, false><<<grid, kThreads, C::SMEM, st>>>(mq, mk, mv, mk64, mv64, p);
  return check_launch();
}

}  // namespace
}  // namespace bsa

#ifdef BSA_TRACE
extern "C" int bsa_trace_dump(void* host, size_t bytes) {
  if (bytes > sizeof(unsigned long long) * (1 << 16)) bytes = sizeof(unsigned long long) * (1 << 16);
  cudaError_t e = cudaMemcpyFromSymbol(host, bsa::g_bsa_trace, bytes);
  return e == cudaSuccess ? BSA_OK : bsa::record_cuda_error(e);
}
#endif

extern "C" size_t bsa_attn_workspace_size(int batch, int heads, int nq, int nk, int block_q,
                                          int block_k, int list_heads) {
  if (batch < 1 || heads < 1 || nq < 1 || nk < 1 || !bsa::block_ok(block_q) ||
      !bsa::block_ok(block_k) || list_heads < 1)
    return 0;
  return bsa::geometry(batch, heads, nq, nk, block_q, block_k, list_heads).total;
}

namespace bsa {
namespace {

// Shared body of bsa_attn_fwd and bsa_attn_fwd_paged.  page_table == nullptr: K/V
// are [batch, nk, heads, head_dim]; else they are one-batch pools of n_pool_pages
// 128-token pages addressed through page_table [batch][pages_per_batch].
// Argument checks of the forward that need no workspace, in the order every
// forward entry point applies them: pointers, sizes, list heads, alignment
// (BSA_ERR_INVALID_ARG), then head_dim and block sizes (BSA_ERR_UNSUPPORTED).
int check_fwd_args(const void* q, const void* k, const void* v, int batch, int heads, int nq,
                   int nk, int head_dim, int qkv_row_stride, int o_row_stride, int block_q,
                   int block_k, const int* row_ptr, const int* col_idx, int list_heads,
                   const void* o, const float* lse) {
  if (!q || !k || !v || !o || !lse || !row_ptr || !col_idx) return BSA_ERR_INVALID_ARG;
  if (batch < 1 || heads < 1 || nq < 1 || nk < 1) return BSA_ERR_INVALID_ARG;
  if (list_heads != 1 && list_heads != batch * heads) return BSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (token_row_stride(qkv_row_stride, heads, head_dim) < 0 ||
      token_row_stride(o_row_stride, heads, head_dim) < 0)
    return BSA_ERR_INVALID_ARG;
  if (!block_ok(block_q) || !block_ok(block_k)) return BSA_ERR_UNSUPPORTED;
  return BSA_OK;
}

int attn_fwd_impl(const void* q, const void* k, const void* v, int batch, int heads, int nq,
                  int nk, int head_dim, int qkv_row_stride, int o_row_stride, int block_q,
                  int block_k, const int* row_ptr, const int* col_idx, int list_heads, float scale,
                  void* o, float* lse, void* ws, size_t ws_bytes, const int* page_table,
                  int pages_per_batch, int n_pool_pages, cudaStream_t st) {
  if (!ws) return BSA_ERR_INVALID_ARG;
  int rc0 = check_fwd_args(q, k, v, batch, heads, nq, nk, head_dim, qkv_row_stride, o_row_stride,
                           block_q, block_k, row_ptr, col_idx, list_heads, o, lse);
  if (rc0 != BSA_OK) return rc0;
  const long long qkv_rs = token_row_stride(qkv_row_stride, heads, head_dim);
  const long long o_rs = token_row_stride(o_row_stride, heads, head_dim);
  // pools of the paged cache are dense [pages * 128, heads, head_dim]
  const long long kv_rs = page_table ? static_cast<long long>(heads) * head_dim : qkv_rs;
  if (!aligned16(ws)) return BSA_ERR_INVALID_ARG;
  if (page_table) {
    // pages hold whole key blocks; a shared list needs a single page table
    if (block_k > kBN || (list_heads == 1 && batch > 1)) return BSA_ERR_UNSUPPORTED;
    if (pages_per_batch < ceil_div(nk, kBN) || n_pool_pages < 1 ||
        static_cast<long long>(n_pool_pages) * kBN > 0x7fffffffLL)
      return BSA_ERR_INVALID_ARG;
  }
  const Geometry g = geometry(batch, heads, nq, nk, block_q, block_k, list_heads);
  if (ws_bytes < g.total) return BSA_ERR_WORKSPACE;
  if (g.nnz_cap > 0x7fffffffLL || static_cast<long long>(ceil_div(nk, kBN)) >= (1LL << 28) ||
      static_cast<long long>(batch) * heads * g.QT > 0x3fffffffLL)
    return BSA_ERR_UNSUPPORTED;
  if (scale <= 0.0f) scale = 1.0f / sqrtf(static_cast<float>(head_dim));

  // 64-token key blocks: tiles are gathered from two arbitrary blocks (64-row boxes)
  const bool gather_k = block_k == 64 && g.KB <= kGatherMaxBlocks;
  CUtensorMap mq, mk, mv, mk64, mv64;
  const int kv_batch = page_table ? 1 : batch;
  const int kv_rows = page_table ? n_pool_pages * kBN : nk;
  if (make_map(&mq, q, batch, nq, heads, head_dim, qkv_rs) != BSA_OK ||
      make_map(&mk, k, kv_batch, kv_rows, heads, head_dim, kv_rs) != BSA_OK ||
      make_map(&mv, v, kv_batch, kv_rows, heads, head_dim, kv_rs) != BSA_OK ||
      make_map(&mk64, k, kv_batch, kv_rows, heads, head_dim, kv_rs, 64) != BSA_OK ||
      make_map(&mv64, v, kv_batch, kv_rows, heads, head_dim, kv_rs, 64) != BSA_OK)
    return BSA_ERR_CUDA;

  char* wsb = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(wsb);
  int* cnt = reinterpret_cast<int*>(wsb + g.cnt_off);
  uint32_t* entries = reinterpret_cast<uint32_t*>(wsb + g.ent_off);
  cudaError_t e = cudaMemsetAsync(status, 0, 2 * sizeof(int), st);  // status word + unit counter
  if (e != cudaSuccess) return record_cuda_error(e);

  int rc = launch_build_lists(row_ptr, col_idx, list_heads, g, nk, block_q, block_k, cnt, entries,
                              status, st, page_table, pages_per_batch, heads, gather_k);
  if (rc != BSA_OK) return rc;

  AttnParams p;
  p.B = batch;
  p.H = heads;
  p.nq = nq;
  p.nk = nk;
  p.QT = g.QT;
  p.block_q = block_q;
  p.block_k = block_k;
  p.QB = g.QB;
  p.LR = g.LR;
  p.list_heads = list_heads;
  p.expand = g.expand;
  p.total_items = batch * heads * g.QT;
  p.total_units = (p.total_items + 1) / 2;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.row_ptr = row_ptr;
  p.cnt = cnt;
  p.entries = entries;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_stride = o_rs;
  p.lse = lse;
  p.status = status;
  p.unit_counter = status + 1;
  p.timeout_ns = 2000000000ULL;
  p.page_table = page_table;
  p.pages_per_batch = pages_per_batch;
  p.gather_k = gather_k ? 1 : 0;
  return head_dim == 128 ? launch_attn<128>(mq, mk, mv, mk64, mv64, p, st)
                         : launch_attn<64>(mq, mk, mv, mk64, mv64, p, st);
}

}  // namespace
}  // namespace bsa

extern "C" int bsa_attn_fwd(const void* q, const void* k, const void* v, int batch, int heads,
                            int nq, int nk, int head_dim, int qkv_row_stride, int o_row_stride,
                            int block_q, int block_k, const int* row_ptr, const int* col_idx,
                            int list_heads, float scale, void* o, float* lse, void* ws,
                            size_t ws_bytes, void* stream) {
  BSA_NVTX_RANGE("bsa_attn_fwd");
  return bsa::attn_fwd_impl(q, k, v, batch, heads, nq, nk, head_dim, qkv_row_stride, o_row_stride,
                            block_q, block_k, row_ptr, col_idx, list_heads, scale, o, lse, ws,
                            ws_bytes, nullptr, 0, 0, static_cast<cudaStream_t>(stream));
}

extern "C" int bsa_attn_fwd_paged(const void* q, const void* k_pool, const void* v_pool,
                                  int n_pool_pages, const int* page_table, int pages_per_batch,
                                  int batch, int heads, int nq, int nk, int head_dim, int block_q,
                                  int block_k, const int* row_ptr, const int* col_idx,
                                  int list_heads, float scale, void* o, float* lse, void* ws,
                                  size_t ws_bytes, void* stream) {
  BSA_NVTX_RANGE("bsa_attn_fwd_paged");
  if (!page_table) return BSA_ERR_INVALID_ARG;
  return bsa::attn_fwd_impl(q, k_pool, v_pool, batch, heads, nq, nk, head_dim, 0, 0, block_q,
                            block_k, row_ptr, col_idx, list_heads, scale, o, lse, ws, ws_bytes,
                            page_table, pages_per_batch, n_pool_pages,
                            static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// Allocation-free variant of bsa_attn_fwd.
//
// Some callers cannot hand the library a workspace: a host framework that owns
// every device byte through its own pre-reserved pool and forbids extra CUDA
// allocations, or a latency-critical serving loop where a cudaMalloc (which may
// synchronise the device) is not allowed.  For them, the attention workspace
// lives in a fixed device array that every GPU loading this library holds until
// the process exits (kNoAllocScratchBytes per device).
// ---------------------------------------------------------------------------
namespace bsa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch in the current device's context, looked up
// with cudaGetSymbolAddress (the host-side name of a __device__ array is only a
// stand-in, never a device address) on the first call made with that device
// current, and again whenever the calling thread's current context is not the one
// the cached address was taken in: after a cudaDeviceReset the module is loaded
// anew and the array may move.  Contexts are told apart by their process-unique
// ids (cuCtxGetId), which a re-created context never repeats.
int noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  static unsigned long long ctx_id_of[64] = {0};
  static PFN_cuCtxGetCurrent_v4000 get_ctx = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_ctx = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
  });
  if (!get_ctx || !get_id) return BSA_ERR_CUDA;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  if (dev < 0 || dev >= 64) return BSA_ERR_UNSUPPORTED;
  // id of the calling thread's current context; 0 when the runtime has not bound
  // one to this thread yet (the symbol lookup below does)
  auto current_id = [&]() -> unsigned long long {
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
  };
  unsigned long long id = current_id();
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev] || id == 0 || ctx_id_of[dev] != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return record_cuda_error(e);
    id = current_id();
    if (id == 0) return BSA_ERR_CUDA;
    addr[dev] = p;
    ctx_id_of[dev] = id;
  }
  *out = addr[dev];
  return BSA_OK;
}

}  // namespace
}  // namespace bsa

extern "C" int bsa_attn_fwd_noalloc(const void* q, const void* k, const void* v, int batch,
                                    int heads, int nq, int nk, int head_dim, int block_q,
                                    int block_k, const int* row_ptr, const int* col_idx,
                                    int list_heads, float scale, void* o, float* lse,
                                    int* device_status, void* stream) {
  BSA_NVTX_RANGE("bsa_attn_fwd_noalloc");
  using namespace bsa;
  // the same argument checks, in the same order, as bsa_attn_fwd before the size check
  int rc = check_fwd_args(q, k, v, batch, heads, nq, nk, head_dim, 0, 0, block_q, block_k,
                          row_ptr, col_idx, list_heads, o, lse);
  if (rc != BSA_OK) return rc;
  const size_t need =
      bsa_attn_workspace_size(batch, heads, nq, nk, block_q, block_k, list_heads);
  if (need == 0) return BSA_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) {
    record_error_message("bsa_attn_fwd_noalloc: this shape needs a larger workspace than the "
                         "library's fixed 8 MiB scratch; use bsa_attn_fwd with a caller workspace");
    return BSA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc != BSA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = bsa_attn_fwd(q, k, v, batch, heads, nq, nk, head_dim, 0, 0, block_q, block_k, row_ptr,
                    col_idx, list_heads, scale, o, lse, scratch, kNoAllocScratchBytes, stream);
  if (rc != BSA_OK || device_status == nullptr) return rc;
  cudaError_t e = cudaMemcpyAsync(device_status, scratch, sizeof(int), cudaMemcpyDeviceToDevice, st);
  return e == cudaSuccess ? BSA_OK : record_cuda_error(e);
}
