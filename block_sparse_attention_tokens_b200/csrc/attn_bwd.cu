// Block-sparse attention backward on sm_100a: dQ, dK, dV over the kept block pairs.
//
// Sources: the Radial explainer (aibr.jp/archives/112136), section 4 (training cost
// cut by the sparse mask), the NABLA explainer (aibr.jp/archives/124678), section 4
// (training and inference speed-up) and the Sparse Forcing summary
// (gist.science/ja/paper/2604.21221): the sparse attention is trained through.
// With P = softmax(S), S = Q K^T * scale restricted to kept block pairs and
// D = rowsum(dO * O):
//     dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  dQ = dS K * scale,  dK = dS^T Q * scale.
// P is recomputed from the forward's log-sum-exp, so nothing else is stored.
//
// Two passes of one kernel template, no atomics:
//   kDKV : one CTA per 128-key tile; iterates the q-tiles that keep it (transposed
//          kept list).  S^T = K Q^T and dP^T = V dO^T (SS MMAs) -> P, dS in registers
//          (thread = key row = TMEM lane) -> bf16 into TMEM -> dV += P dO and
//          dK += dS Q (TS MMAs, A operand from TMEM).
//   kDQ  : one CTA per 128-row q-tile; iterates its kept list.  S = Q K^T and
//          dP = dO V^T -> dS -> dQ += dS K.
// TMEM: S | dP (128 columns each, fp32), accA (dK or dQ) and accB (dV).  The
// compute warps turn S and dP into P and dS (bf16, packed over the columns they
// were read from) in two 64-column halves and publish each half on its own: the
// MMA warp accumulates the first half while the second is computed, then issues
// the next step's S and dP.  Warps 0-7 compute (two per TMEM lane quarter, 32
// columns of each half), warp 8 feeds a ring of 128-row operand tiles with TMA,
// warp 9 issues the MMAs.  Units are handed out from a global counter through a
// shared-memory ring as in the forward kernel.  All waits are bounded.
#include "bsa_common.cuh"
#include "tmem_io.cuh"
#include "attn_common.cuh"
#include "nvtx_range.cuh"

namespace bsa {
namespace {

// Optional per-step timeline of CTA 0 of the dK/dV pass (SM clock), compiled only
// with -DBSA_TRACE and read back with bsa_btrace_dump().
#ifdef BSA_TRACE
__device__ unsigned long long g_bsa_btrace[1 << 16];
#define BSA_BTRACE_AT(step, slot)                                                      \
  do {                                                                                 \
    if (kDKV && blockIdx.x == 0 && (step) < (1 << 13)) g_bsa_btrace[(step) * 8 + (slot)] = clock64(); \
  } while (0)
#else
#define BSA_BTRACE_AT(step, slot) \
  do {                            \
  } while (0)
#endif

constexpr int kBwdThreads = 320;
// BSA_BWD_LOAD_ALL=1: the decoupled passes load S (and dP) of both 64-column halves
// before computing either (one exposed load latency per entry, at the price of
// more live registers); 0: one half at a time.
#ifndef BSA_BWD_LOAD_ALL
#define BSA_BWD_LOAD_ALL 0
#endif
constexpr bool kLoadAll = BSA_BWD_LOAD_ALL != 0;
constexpr int kBwdLoadWarp = 8;
constexpr int kBwdMmaWarp = 9;

// The fused dK/dV pass hands P and dS to the accumulation MMAs in four 32-query
// quarters, so the tensor pipe starts on an entry's accumulation after a quarter of
// its compute (an SM-clock trace: 458 instead of 863 cycles from S to the first
// accumulation, 8.6 % shorter entries); BSA_BWD_QUARTERS=0 builds the two 64-query
// halves instead.
#ifndef BSA_BWD_QUARTERS
#define BSA_BWD_QUARTERS 1
#endif
constexpr bool kQuarters = BSA_BWD_QUARTERS != 0;

// 16-column TMEM load without its wait (the quarter-granular compute issues the
// loads of S and dP back to back and waits once, tying both destinations)
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                 "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
               : "r"(taddr)
               : "memory");
}

template <int D>
struct BwdCfg {
  static constexpr int KCH = D / 64;
  static constexpr int CHUNK_BYTES = kBM * 128;          // 128 rows of one 64-column chunk
  static constexpr int TILE_BYTES = KCH * CHUNK_BYTES;   // 128 rows x D bf16
  // ring of single operand tiles (colA, colB alternating): as deep as shared memory
  // allows, a tile load takes several steps of MMA time to arrive
  static constexpr int NSTAGE = D == 128 ? 5 : 10;
  static constexpr int OFF_ROW = 0;                      // the two row-operand tiles
  static constexpr int OFF_RING = 2 * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_RING + NSTAGE * TILE_BYTES;
  static constexpr int SMEM = OFF_BAR + 512 + 1024;
};

struct BwdParams {
  int B, H, nq, nk, QT, KT;
  int list_heads, LR, QB, expand, block_q;
  int total_items;
  float scale, scale_log2;
  const int* row_ptr;
  const int* cnt;
  const uint32_t* entries;   // forward per-q-tile lists
  const int* tcnt;
  const uint32_t* tentries;  // transposed per-k-tile lists, stride QT
  const float* lse2;         // [B*H][QT*128]: LSE * log2(e), +inf past nq / for empty rows
  const float* dvec;         // [B*H][QT*128]: rowsum(dO * O), 0 past nq
  __nv_bfloat16* outA;       // dK (kDKV) or dQ (kDQ)
  __nv_bfloat16* outB;       // dV (kDKV)
  long long out_stride;      // elements between consecutive token rows of outA / outB
  int* status;
  int* unit_counter;
  unsigned long long timeout_ns;
};

struct BItem {
  int b, h, row_tile, n;     // n < 0: none
  const uint32_t* ent;
};

// Kernel passes.  kPassDKV: dK and dV together (two accumulators, P and dS written
// over the S and dP columns, so each entry's accumulation precedes the next
// entry's S and dP).  The decoupled passes hold one accumulator and put the
// accumulation operand (dS or P, bf16) in a double-buffered region of the free
// TMEM columns [384, 512), so the next entry's S (and dP) are issued as soon as
// the current ones have been read:
//   kPassDQ: rows = q-tiles,   S = Q K^T, dP = dO V^T, dQ += dS K
//   kPassDK: rows = key tiles, S = K Q^T, dP = V dO^T, dK += dS Q
//   kPassDV: rows = key tiles, S = K Q^T,              dV += P dO
enum : int { kPassDKV = 0, kPassDQ = 1, kPassDK = 2, kPassDV = 3 };

template <int kPass>
struct PassTraits {
  static constexpr bool kKeyRows = kPass != kPassDQ;      // items are key tiles
  static constexpr bool kFused = kPass == kPassDKV;
  static constexpr bool kHasDP = kPass != kPassDV;        // dP (and the second row operand)
  static constexpr bool kAccColB = kPass == kPassDV;      // accumulate with colB (dO)
};

template <bool kDKV>
__device__ __forceinline__ BItem get_bitem(const BwdParams& p, int it) {
  BItem r;
  r.n = -1;
  r.ent = nullptr;
  r.b = r.h = r.row_tile = 0;
  if (it >= p.total_items) return r;
  const int per = kDKV ? p.KT : p.QT;
  r.row_tile = it % per;
  const int bh = it / per;
  r.h = bh % p.H;
  r.b = bh / p.H;
  const int mh = p.list_heads == 1 ? 0 : bh;
  if (kDKV) {
    const long long g = static_cast<long long>(mh) * p.KT + r.row_tile;
    r.n = p.tcnt[g];
    r.ent = p.tentries + g * p.QT;
  } else {
    const int lr = p.block_q >= 128 ? (r.row_tile * kBM) / p.block_q : r.row_tile;
    const int first_qb = p.block_q >= 128 ? lr : 2 * lr;
    r.n = p.cnt[mh * p.LR + lr];
    r.ent = p.entries + static_cast<long long>(p.row_ptr[mh * p.QB + first_qb]) * p.expand;
  }
  return r;
}

// rowA / rowB: the item's fixed operands (key-row passes: K, V; dQ pass: Q, dO;
// the dV pass uses rowA only), 128-row tiles.  colA / colB: the per-step operands
// (key-row passes: Q, dO; dQ pass: K, V), 128-row tiles streamed through the ring
// (colA then colB per kept entry).
template <int D, int kPass>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tmRowA, const __grid_constant__ CUtensorMap tmRowB,
                    const __grid_constant__ CUtensorMap tmColA, const __grid_constant__ CUtensorMap tmColB,
                    const BwdParams p) {
  using C = BwdCfg<D>;
  using T = PassTraits<kPass>;
  constexpr bool kDKV = T::kKeyRows;   // per-column LSE / Delta, transposed lists
  constexpr int kRowTiles = T::kHasDP ? 2 : 1;
  // ring order per entry: colB before colA when the accumulation holds colA
  constexpr bool kLoadHeldLast = !T::kFused && !T::kAccColB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sRow = sbase + C::OFF_ROW;
  const uint32_t sRing = sbase + C::OFF_RING;
  const uint32_t bar0 = smem_u32(smem + C::OFF_BAR);
  auto FULL = [&](int i) { return bar0 + 8u * i; };
  auto EMPTY = [&](int i) { return bar0 + 8u * (C::NSTAGE + i); };
  const uint32_t ROWFULL = bar0 + 8u * (2 * C::NSTAGE + 0);
  const uint32_t ROWEMPTY = bar0 + 8u * (2 * C::NSTAGE + 1);
  const uint32_t SFULL = bar0 + 8u * (2 * C::NSTAGE + 2);
  auto PREADY = [&](int half) { return bar0 + 8u * (2 * C::NSTAGE + 3 + half); };
  // quarters 0, 1 share the halves' barriers; 2, 3 follow the TMEM slot words
  auto PREADYQ = [&](int q) {
    return q < 2 ? PREADY(q) : bar0 + 8u * (2 * C::NSTAGE + 21 + (q - 2));
  };
  const uint32_t DONE = bar0 + 8u * (2 * C::NSTAGE + 5);
  const uint32_t FINAL = bar0 + 8u * (2 * C::NSTAGE + 6);
  auto UFULL = [&](int i) { return bar0 + 8u * (2 * C::NSTAGE + 7 + i); };
  auto UEMPTY = [&](int i) { return bar0 + 8u * (2 * C::NSTAGE + 11 + i); };
  // decoupled passes: S (and dP) of the current entry read by every compute warp
  // (the next entry's may be issued), and buffer b read by its accumulation MMAs
  // (free to refill); PREADY(b) then signals "the entry's dS or P is in buffer b"
  const uint32_t SREAD = bar0 + 8u * (2 * C::NSTAGE + 15);
  auto DSFREE = [&](int b) { return bar0 + 8u * (2 * C::NSTAGE + 16 + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 8 * (2 * C::NSTAGE + 18));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(FULL(i), 1);
      mbar_init(EMPTY(i), 1);
    }
    mbar_init(ROWFULL, 1);
    mbar_init(ROWEMPTY, 1);
    mbar_init(SFULL, 1);
    mbar_init(PREADY(0), 8);
    mbar_init(PREADY(1), 8);
    if (kQuarters) {
      mbar_init(PREADYQ(2), 8);
      mbar_init(PREADYQ(3), 8);
    }
    mbar_init(DONE, 1);
    mbar_init(FINAL, 1);
    mbar_init(SREAD, 8);
    mbar_init(DSFREE(0), 1);
    mbar_init(DSFREE(1), 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(UFULL(i), 1);
      mbar_init(UEMPTY(i), 1 + 8);  // MMA thread + 8 compute warps
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == kBwdMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kBwdLoadWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int st = 0;
      uint32_t ph = 0, rph = 0;
      uint32_t filled = 0, fill_phase = 0;
      int row_filled = -1;
      bool ok = true;
      uint32_t gl = 0;  // steps loaded (trace index)
      (void)gl;
      auto load_col = [&](const CUtensorMap* map, const BItem& it, int ct) -> bool {
        if (!mbar_wait(EMPTY(st), ph ^ 1u, abort_flag, p.status, p.timeout_ns)) return false;
        mbar_expect_tx(FULL(st), C::TILE_BYTES);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(sRing + st * C::TILE_BYTES + c * C::CHUNK_BYTES, map, FULL(st), 64 * c,
                      it.h, ct * kBM, it.b);
        filled |= 1u << st;
        fill_phase = (fill_phase & ~(1u << st)) | (ph << st);
        if (++st == C::NSTAGE) { st = 0; ph ^= 1u; }
        return true;
      };
      for (int uk = 0; ok; ++uk) {
        const int slot = uk & 3;
        if (!mbar_wait(UEMPTY(slot), ((uk >> 2) & 1) ^ 1u, abort_flag, p.status, p.timeout_ns)) {
          ok = false;
          break;
        }
        const int u = atomicAdd(p.unit_counter, 1);
        unit_ring[slot] = u;
        mbar_arrive(UFULL(slot));
        if (u >= p.total_items) break;
        const BItem it = get_bitem<kDKV>(p, u);
        if (it.n <= 0) continue;
        if (!mbar_wait(ROWEMPTY, rph ^ 1u, abort_flag, p.status, p.timeout_ns)) {
          ok = false;
          break;
        }
        row_filled = static_cast<int>(rph);
        rph ^= 1u;
        mbar_expect_tx(ROWFULL, kRowTiles * C::TILE_BYTES);
        for (int c = 0; c < C::KCH; ++c) {
          tma_load_4d(sRow + c * C::CHUNK_BYTES, &tmRowA, ROWFULL, 64 * c, it.h,
                      it.row_tile * kBM, it.b);
          if (kRowTiles == 2)
            tma_load_4d(sRow + C::TILE_BYTES + c * C::CHUNK_BYTES, &tmRowB, ROWFULL, 64 * c, it.h,
                        it.row_tile * kBM, it.b);
        }
        // entry words read four ahead, so no load latency sits between two TMA issues
        uint32_t pf0 = __ldg(it.ent), pf1 = it.n > 1 ? __ldg(it.ent + 1) : 0u;
        uint32_t pf2 = it.n > 2 ? __ldg(it.ent + 2) : 0u, pf3 = it.n > 3 ? __ldg(it.ent + 3) : 0u;
        for (int j = 0; j < it.n && ok; ++j) {
          const uint32_t ent = pf0;
          pf0 = pf1;
          pf1 = pf2;
          pf2 = pf3;
          pf3 = j + 4 < it.n ? __ldg(it.ent + j + 4) : 0u;
          const int ct = static_cast<int>(ent & 0x0FFFFFFFu);
          // decoupled passes: the operand released early (after S / dP) first, the
          // one the accumulation holds second -- in the ring the next entry's early
          // operand then reuses the stage of an operand released an entry sooner,
          // which gives the loads one more entry of lead
          if (kLoadHeldLast) {
            ok = load_col(&tmColB, it, ct);
            ok = ok && load_col(&tmColA, it, ct);
          } else {
            ok = load_col(&tmColA, it, ct);
            ok = ok && load_col(&tmColB, it, ct);
          }
          BSA_BTRACE_AT(gl, 7);
          ++gl;
        }
      }
      for (int i = 0; i < C::NSTAGE; ++i)
        if (filled & (1u << i))
          mbar_wait_drain(FULL(i), (fill_phase >> i) & 1u, p.status, p.timeout_ns);
      if (row_filled >= 0)
        mbar_wait_drain(ROWFULL, static_cast<uint32_t>(row_filled), p.status, p.timeout_ns);
    }
  } else if (warp == kBwdMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_ss = idesc_bf16_f32(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_ts = idesc_bf16_f32(kBM, D, 0, 1);
      constexpr uint32_t kTileUnits = C::TILE_BYTES >> 4;
      const uint64_t dRowK = smem_desc_sw128(sRow, 16, 1024);
      const uint64_t dColK = smem_desc_sw128(sRing, 16, 1024);
      const uint64_t dColMN = smem_desc_sw128(sRing, C::CHUNK_BYTES, 1024);
      int st = 0;
      uint32_t ph = 0, rph = 0, pph = 0;
      bool ok = true;
      uint32_t gm = 0;  // steps issued (trace index)
      (void)gm;
      auto acquire = [&](int& stage) -> bool {
        if (!mbar_wait(FULL(st), ph, abort_flag, p.status, p.timeout_ns)) return false;
        stage = st;
        if (++st == C::NSTAGE) { st = 0; ph ^= 1u; }
        return true;
      };
      // S-like = rowA colA^T into TMEM [0,128), dP-like = rowB colB^T into [128,256)
      auto sd = [&](int sa, int sb) {
        tc_fence_after();
        const uint64_t da = dColK + static_cast<uint64_t>(sa * kTileUnits);
        const uint64_t db = dColK + static_cast<uint64_t>(sb * kTileUnits);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off =
              static_cast<uint64_t>((((kk >> 2) * C::CHUNK_BYTES) + (kk & 3) * 32) >> 4);
          mma_ss(tmem, dRowK + off, da + off, idesc_ss, kk > 0 ? 1u : 0u);
        }
        if constexpr (T::kHasDP) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off =
                static_cast<uint64_t>((((kk >> 2) * C::CHUNK_BYTES) + (kk & 3) * 32) >> 4);
            mma_ss(tmem + 128, dRowK + kTileUnits + off, db + off, idesc_ss, kk > 0 ? 1u : 0u);
          }
        }
      };
      // one 64-column half of the accumulation: accA (+)= dS colA, accB (+)= P colB
      // (kDKV); packed bf16 columns 16*kk .. of P / dS sit at TMEM column
      // (kk / 2) * 32 + (kk % 2) * 8 of their half (each compute warp packs its 32
      // columns into the first 16 of its own)
      auto acc = [&](int sa, int sb, int half, bool first) {
        tc_fence_after();
        const uint64_t dA = dColMN + static_cast<uint64_t>(sa * kTileUnits);
        const uint64_t dB = dColMN + static_cast<uint64_t>(sb * kTileUnits);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = half * 4 + k4;
          const uint32_t col = half * 64 + (k4 >> 1) * 32 + (k4 & 1) * 8;
          const uint32_t a0 = (first && k4 == 0) ? 0u : 1u;
          mma_ts(tmem + 256, tmem + 128 + col, dA + static_cast<uint64_t>(kk * 128), idesc_ts, a0);
          if (kDKV)
            mma_ts(tmem + 256 + D, tmem + col, dB + static_cast<uint64_t>(kk * 128), idesc_ts,
                   a0);
        }
      };
      // one 32-query quarter of the accumulation: warp group cg packed queries
      // 32q + 16cg .. + 15 into TMEM columns 32q + 16cg .. + 7
      auto acc_q = [&](int sa, int sb, int q, bool first) {
        tc_fence_after();
        const uint64_t dA = dColMN + static_cast<uint64_t>(sa * kTileUnits);
        const uint64_t dB = dColMN + static_cast<uint64_t>(sb * kTileUnits);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const int kk = 2 * q + g;
          const uint32_t col = 32 * q + 16 * g;
          const uint32_t a0 = (first && g == 0) ? 0u : 1u;
          mma_ts(tmem + 256, tmem + 128 + col, dA + static_cast<uint64_t>(kk * 128), idesc_ts, a0);
          mma_ts(tmem + 256 + D, tmem + col, dB + static_cast<uint64_t>(kk * 128), idesc_ts, a0);
        }
      };
      (void)acc_q;
      // dQ pass: dQ += dS K with dS from a double-buffered region of the free TMEM
      // columns [384, 512), so S and dP of the next entry are issued as soon as the
      // compute warps have read the current ones (SREAD), ahead of this entry's dQ
      // MMAs; K stays resident until its dQ MMAs, V is released after dP.
      uint32_t g_sd = 0, g_acc = 0;  // S/dP pairs issued / dQ accumulations issued (whole CTA)
      auto issue_sd = [&](int sa, int sb) -> bool {
        // S/dP TMEM may be overwritten once the previous entry's S/dP have been read
        if (g_sd > 0 && !mbar_wait(SREAD, (g_sd - 1) & 1u, abort_flag, p.status, p.timeout_ns))
          return false;
        sd(sa, sb);
        mma_commit(SFULL);
        mma_commit(EMPTY(T::kAccColB ? sa : sb));   // the operand the accumulation does not read
        ++g_sd;
        return true;
      };
      // acc (+)= buffer . (colA or colB); `sacc` is the ring stage of that operand
      auto acc_dq = [&](int sacc, bool first) {
        tc_fence_after();
        const uint32_t buf = g_acc & 1u;
        const uint64_t dA = dColMN + static_cast<uint64_t>(sacc * kTileUnits);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + 256, tmem + 384 + 64 * buf + 8 * kk, dA + static_cast<uint64_t>(kk * 128),
                 idesc_ts, (first && kk == 0) ? 0u : 1u);
      };
      for (int uk = 0; ok; ++uk) {
        const int slot = uk & 3;
        if (!mbar_wait(UFULL(slot), (uk >> 2) & 1, abort_flag, p.status, p.timeout_ns)) {
          ok = false;
          break;
        }
        const int u = unit_ring[slot];
        mbar_arrive(UEMPTY(slot));
        if (u >= p.total_items) break;
        const BItem it = get_bitem<kDKV>(p, u);
        if (it.n <= 0) continue;
        if (!mbar_wait(ROWFULL, rph, abort_flag, p.status, p.timeout_ns)) {
          ok = false;
          break;
        }
        rph ^= 1u;
        int sa = 0, sb = 0;
        if (kLoadHeldLast ? (!acquire(sb) || !acquire(sa)) : (!acquire(sa) || !acquire(sb))) {
          ok = false;
          break;
        }
        if constexpr (!T::kFused) {
          if (!issue_sd(sa, sb)) { ok = false; break; }
          if (it.n == 1) mma_commit(ROWEMPTY);
          int sacc = T::kAccColB ? sb : sa;
          for (int j = 0; j < it.n && ok; ++j) {
            int na = 0, nb = 0;
            if (j + 1 < it.n) {
              const bool got = kLoadHeldLast ? (acquire(nb) && acquire(na)) : (acquire(na) && acquire(nb));
              if (!got || !issue_sd(na, nb)) { ok = false; break; }
              if (j + 2 == it.n) mma_commit(ROWEMPTY);
            }
            const uint32_t buf = g_acc & 1u;
            if (!mbar_wait(PREADY(buf), (g_acc >> 1) & 1u, abort_flag, p.status, p.timeout_ns)) {
              ok = false;
              break;
            }
            acc_dq(sacc, j == 0);
            mma_commit(EMPTY(sacc));
            mma_commit(DSFREE(buf));
            ++g_acc;
            if (j == it.n - 1) mma_commit(DONE);
            sacc = T::kAccColB ? nb : na;
          }
          continue;
        }
        sd(sa, sb);
        mma_commit(SFULL);
        if (it.n == 1) mma_commit(ROWEMPTY);
        for (int j = 0; j < it.n && ok; ++j) {
          if constexpr (kQuarters && kDKV) {
            for (int q = 0; q < 4; ++q) {
              if (!mbar_wait(PREADYQ(q), pph, abort_flag, p.status, p.timeout_ns)) {
                ok = false;
                break;
              }
              if (q == 0 || q == 3) BSA_BTRACE_AT(gm, 4 + (q == 3));
              acc_q(sa, sb, q, j == 0 && q == 0);
            }
          } else {
          for (int half = 0; half < 2; ++half) {
            if (!mbar_wait(PREADY(half), pph, abort_flag, p.status, p.timeout_ns)) {
              ok = false;
              break;
            }
            BSA_BTRACE_AT(gm, 4 + half);
            acc(sa, sb, half, j == 0 && half == 0);
          }
          }
          if (!ok) break;
          pph ^= 1u;
          mma_commit(EMPTY(sa));
          mma_commit(EMPTY(sb));
          ++gm;
          if (j == it.n - 1) {
            mma_commit(DONE);
          } else {
            if (!acquire(sa) || !acquire(sb)) { ok = false; break; }
            BSA_BTRACE_AT(gm, 6);
            sd(sa, sb);
            mma_commit(SFULL);
            if (j + 1 == it.n - 1) mma_commit(ROWEMPTY);
          }
        }
      }
      mma_commit(FINAL);
      mbar_wait_drain(FINAL, 0, p.status, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ compute (8 warps)
    const int q4 = warp & 3;            // TMEM lane quarter
    const int cg = warp >> 2;           // column group: columns 32*cg .. +31 of each half
    const int row = q4 * 32 + lane;     // 0..127 = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t tA = tmem + lane_base + 256;
    const uint32_t tB = tmem + lane_base + 256 + D;
    const int rh = q4 >> 1;  // which 64-row half of the row tile (warp-uniform)
    const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
    uint32_t sph = 0, dph = 0;
    bool ok = true;
    uint32_t gc = 0;  // steps computed (trace index)
    (void)gc;
    for (int uk = 0; ok; ++uk) {
      const int slot = uk & 3;
      if (!mbar_wait(UFULL(slot), (uk >> 2) & 1, abort_flag, p.status, p.timeout_ns)) {
        ok = false;
        break;
      }
      const int u = unit_ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(UEMPTY(slot));
      if (u >= p.total_items) break;
      const BItem it = get_bitem<kDKV>(p, u);
      if (it.n < 0) continue;
      const long long bh = static_cast<long long>(it.b) * p.H + it.h;
      const int grow = it.row_tile * kBM + row;          // global row of this thread
      const float* lse2_bh = p.lse2 + bh * (p.QT * kBM);
      const float* dvec_bh = p.dvec + bh * (p.QT * kBM);
      float2 nlse = make_float2(0.f, 0.f), dd = make_float2(0.f, 0.f);
      if (!kDKV) {
        const float l = -lse2_bh[grow];
        const float d = dvec_bh[grow];
        nlse = make_float2(l, l);
        dd = make_float2(d, d);
      }
      // register prefetch, one entry ahead: the entry word and (kDKV) this lane's
      // -LSE2 / D values of column 64*h + 32*cg + lane, broadcast to the warp by
      // shuffles when used
      uint32_t ent_next = it.n > 0 ? __ldg(it.ent) : 0u;
      // column (query) whose statistics lane `lane` holds in slot h: halves (64h +
      // 32cg + lane), or quarters (32 (2h + lane / 16) + 16cg + lane % 16)
      const int stat_col0 = (kQuarters && kDKV) ? 32 * (lane >> 4) + 16 * cg + (lane & 15)
                                                : 32 * cg + lane;
      constexpr int stat_step = 64;
      float pl[2] = {0.f, 0.f}, pd[2] = {0.f, 0.f};
      if (kDKV && it.n > 0) {
        const int ct0 = static_cast<int>(ent_next & 0x0FFFFFFFu);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          pl[h] = -__ldg(lse2_bh + ct0 * kBM + stat_step * h + stat_col0);
          pd[h] = __ldg(dvec_bh + ct0 * kBM + stat_step * h + stat_col0);
        }
      }
      for (int j = 0; j < it.n && ok; ++j) {
        const uint32_t ent = ent_next;
        const int ct = static_cast<int>(ent & 0x0FFFFFFFu);
        const uint32_t bits = ent >> 28;
        if (j + 1 < it.n) ent_next = __ldg(it.ent + j + 1);
        float cl[2] = {pl[0], pl[1]}, cd[2] = {pd[0], pd[1]};
        if (kDKV && j + 1 < it.n) {
          const int ctn = static_cast<int>(ent_next & 0x0FFFFFFFu);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            pl[h] = -__ldg(lse2_bh + ctn * kBM + stat_step * h + stat_col0);
            pd[h] = __ldg(dvec_bh + ctn * kBM + stat_step * h + stat_col0);
          }
        }
        // keys past nk in the dQ pass (ragged last key tile) are masked per column
        const int cvalid = kDKV ? kBN : p.nk - ct * kBN;
        if (threadIdx.x == 0) BSA_BTRACE_AT(gc, 0);
        ok = mbar_wait(SFULL, sph, abort_flag, p.status, p.timeout_ns);
        if (!ok) break;
        if (threadIdx.x == 0) BSA_BTRACE_AT(gc, 1);
        sph ^= 1u;
        tc_fence_after();
        if constexpr (!T::kFused) {
          // dS (or P) of this entry goes to buffer gc & 1 of the free TMEM columns;
          // the buffer's previous contents must have been consumed by their MMAs
          const uint32_t buf = gc & 1u;
          if (gc >= 2) {
            ok = mbar_wait(DSFREE(buf), ((gc >> 1) - 1) & 1u, abort_flag, p.status, p.timeout_ns);
            if (!ok) break;
            tc_fence_after();
          }
          const uint32_t tD = tmem + lane_base + 384 + 64 * buf + 16 * cg;
          if constexpr (kLoadAll) {
          // S (and dP) of both halves are loaded at once: one load latency per
          // entry, and the next entry's S / dP may be issued as soon as they are in
          // registers
          uint32_t sr[2][32], dr[2][32];
          bool hok[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            hok[h] = (bits >> (rh * 2 + h)) & 1u;
            const uint32_t tS = tmem + lane_base + 64u * h + 32u * cg;
            if (hok[h]) {
              tmem_ld32x32b_x32_nowait(tS, sr[h]);
              if constexpr (T::kHasDP) tmem_ld32x32b_x32_nowait(tS + 128, dr[h]);
            }
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (hok[h]) {
              tmem_wait_ld_x32(sr[h]);
              if constexpr (T::kHasDP) tmem_wait_ld_x32(dr[h]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(SREAD);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t dpk[16];
            if (!hok[h]) {
#pragma unroll
              for (int i = 0; i < 16; ++i) dpk[i] = 0u;
            } else {
              const int cbase = 64 * h + 32 * cg;
              const float vl = h ? cl[1] : cl[0], vd = h ? cd[1] : cd[0];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int c = cbase + 2 * i;
                float2 nl = nlse, dv = dd;
                if constexpr (T::kKeyRows) {  // per-column (query) statistics
                  nl = make_float2(__shfl_sync(0xffffffffu, vl, 2 * i),
                                   __shfl_sync(0xffffffffu, vl, 2 * i + 1));
                  if constexpr (T::kHasDP)
                    dv = make_float2(__shfl_sync(0xffffffffu, vd, 2 * i),
                                     __shfl_sync(0xffffffffu, vd, 2 * i + 1));
                }
                const float2 a = ffma2(make_float2(__uint_as_float(sr[h][2 * i]),
                                                   __uint_as_float(sr[h][2 * i + 1])), sl2, nl);
                float2 pr = make_float2(fast_exp2(a.x), fast_exp2(a.y));
                if constexpr (!T::kKeyRows) {   // dQ pass: ragged key tail
                  if (c >= cvalid) pr.x = 0.f;
                  if (c + 1 >= cvalid) pr.y = 0.f;
                }
                float2 val = pr;
                if constexpr (T::kHasDP)
                  val = fmul2(pr, fsub2(make_float2(__uint_as_float(dr[h][2 * i]),
                                                    __uint_as_float(dr[h][2 * i + 1])),
                                        dv));
                __nv_bfloat162 hd = __floats2bfloat162_rn(val.x, val.y);
                dpk[i] = *reinterpret_cast<uint32_t*>(&hd);
              }
            }
            tmem_st32x32b_x16(tD + 32 * h, dpk);
          }
          } else {
          for (int h = 0; h < 2; ++h) {
            const uint32_t tS = tmem + lane_base + 64u * h + 32u * cg;
            const bool row_ok = (bits >> (rh * 2 + h)) & 1u;
            uint32_t dpk[16];
            uint32_t sr[32], dr[32];
            if (row_ok) {
              tmem_ld32x32b_x32_nowait(tS, sr);
              if constexpr (T::kHasDP) tmem_ld32x32b_x32_nowait(tS + 128, dr);
              tmem_wait_ld_x32(sr);
              if constexpr (T::kHasDP) tmem_wait_ld_x32(dr);
            }
            if (h == 1) {  // S and dP of this entry are in registers: the next may be issued
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(SREAD);
            }
            if (!row_ok) {
#pragma unroll
              for (int i = 0; i < 16; ++i) dpk[i] = 0u;
            } else {
              const int cbase = 64 * h + 32 * cg;
              const float vl = h ? cl[1] : cl[0], vd = h ? cd[1] : cd[0];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int c = cbase + 2 * i;
                float2 nl = nlse, dv = dd;
                if constexpr (T::kKeyRows) {  // per-column (query) statistics
                  nl = make_float2(__shfl_sync(0xffffffffu, vl, 2 * i),
                                   __shfl_sync(0xffffffffu, vl, 2 * i + 1));
                  if constexpr (T::kHasDP)
                    dv = make_float2(__shfl_sync(0xffffffffu, vd, 2 * i),
                                     __shfl_sync(0xffffffffu, vd, 2 * i + 1));
                }
                const float2 a = ffma2(make_float2(__uint_as_float(sr[2 * i]),
                                                   __uint_as_float(sr[2 * i + 1])), sl2, nl);
                float2 pr = make_float2(fast_exp2(a.x), fast_exp2(a.y));
                if constexpr (!T::kKeyRows) {   // dQ pass: ragged key tail
                  if (c >= cvalid) pr.x = 0.f;
                  if (c + 1 >= cvalid) pr.y = 0.f;
                }
                float2 val = pr;
                if constexpr (T::kHasDP)
                  val = fmul2(pr, fsub2(make_float2(__uint_as_float(dr[2 * i]),
                                                    __uint_as_float(dr[2 * i + 1])),
                                        dv));
                __nv_bfloat162 hd = __floats2bfloat162_rn(val.x, val.y);
                dpk[i] = *reinterpret_cast<uint32_t*>(&hd);
              }
            }
            tmem_st32x32b_x16(tD + 32 * h, dpk);
          }
          }
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(PREADY(buf));
        } else if constexpr (kQuarters && kDKV) {
        for (int q = 0; q < 4; ++q) {
          // this warp's 16 columns of the quarter (queries 32q + 16cg ..); P and dS
          // are packed into the first 8 columns of the same ranges of S and dP
          const uint32_t tS = tmem + lane_base + 32u * q + 16u * cg;
          const bool row_ok = (bits >> (rh * 2 + (q >> 1))) & 1u;
          if (!row_ok) {
            uint32_t z[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) z[i] = 0u;
            tmem_st32x32b_x8(tS, z);
            tmem_st32x32b_x8(tS + 128, z);
          } else {
            uint32_t sd[32];   // S in [0, 16), dP in [16, 32)
            tmem_ld16_nowait(tS, sd);
            tmem_ld16_nowait(tS + 128, sd + 16);
            tmem_wait_ld_x32(sd);
            const float vl = cl[q >> 1], vd = cd[q >> 1];
            const int src0 = (q & 1) << 4;
            uint32_t ppk[8], dpk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 nl = make_float2(__shfl_sync(0xffffffffu, vl, src0 + 2 * i),
                                            __shfl_sync(0xffffffffu, vl, src0 + 2 * i + 1));
              const float2 dv = make_float2(__shfl_sync(0xffffffffu, vd, src0 + 2 * i),
                                            __shfl_sync(0xffffffffu, vd, src0 + 2 * i + 1));
              const float2 a = ffma2(make_float2(__uint_as_float(sd[2 * i]),
                                                 __uint_as_float(sd[2 * i + 1])), sl2, nl);
              const float2 pr = make_float2(fast_exp2(a.x), fast_exp2(a.y));
              const float2 ds = fmul2(pr, fsub2(make_float2(__uint_as_float(sd[16 + 2 * i]),
                                                            __uint_as_float(sd[16 + 2 * i + 1])),
                                                dv));
              __nv_bfloat162 hp = __floats2bfloat162_rn(pr.x, pr.y);
              __nv_bfloat162 hd = __floats2bfloat162_rn(ds.x, ds.y);
              ppk[i] = *reinterpret_cast<uint32_t*>(&hp);
              dpk[i] = *reinterpret_cast<uint32_t*>(&hd);
            }
            tmem_st32x32b_x8(tS, ppk);
            tmem_st32x32b_x8(tS + 128, dpk);
          }
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          tc_fence_before();
          __syncwarp();
          if (threadIdx.x == 0 && (q == 0 || q == 3)) BSA_BTRACE_AT(gc, 2 + (q == 3));
          if (lane == 0) mbar_arrive(PREADYQ(q));
        }
        } else {
        for (int h = 0; h < 2; ++h) {
          // this warp's 32 columns of the half; P and dS are packed into the first 16
          // columns of the same ranges of S and dP
          const uint32_t tS = tmem + lane_base + 64u * h + 32u * cg;
          const bool row_ok = (bits >> (rh * 2 + h)) & 1u;
          if (!row_ok) {
            uint32_t z[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) z[i] = 0u;
            tmem_st32x32b_x16(tS, z);
            tmem_st32x32b_x16(tS + 128, z);
          } else {
            uint32_t sr[32], dr[32];
            tmem_ld32x32b_x32_nowait(tS, sr);
            tmem_ld32x32b_x32_nowait(tS + 128, dr);
            tmem_wait_ld_x32(sr);
            tmem_wait_ld_x32(dr);
            const int cbase = 64 * h + 32 * cg;
            const float vl = h ? cl[1] : cl[0], vd = h ? cd[1] : cd[0];
            uint32_t ppk[16], dpk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int c = cbase + 2 * i;
              float2 nl = nlse, dv = dd;
              if (kDKV) {
                nl = make_float2(__shfl_sync(0xffffffffu, vl, 2 * i),
                                 __shfl_sync(0xffffffffu, vl, 2 * i + 1));
                dv = make_float2(__shfl_sync(0xffffffffu, vd, 2 * i),
                                 __shfl_sync(0xffffffffu, vd, 2 * i + 1));
              }
              const float2 a = ffma2(make_float2(__uint_as_float(sr[2 * i]),
                                                 __uint_as_float(sr[2 * i + 1])), sl2, nl);
              float2 pr = make_float2(fast_exp2(a.x), fast_exp2(a.y));
              if (!kDKV) {
                if (c >= cvalid) pr.x = 0.f;
                if (c + 1 >= cvalid) pr.y = 0.f;
              }
              const float2 ds = fmul2(pr, fsub2(make_float2(__uint_as_float(dr[2 * i]),
                                                            __uint_as_float(dr[2 * i + 1])),
                                                dv));
              __nv_bfloat162 hp = __floats2bfloat162_rn(pr.x, pr.y);
              __nv_bfloat162 hd = __floats2bfloat162_rn(ds.x, ds.y);
              ppk[i] = *reinterpret_cast<uint32_t*>(&hp);
              dpk[i] = *reinterpret_cast<uint32_t*>(&hd);
            }
            if (kDKV) tmem_st32x32b_x16(tS, ppk);
            tmem_st32x32b_x16(tS + 128, dpk);
          }
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          tc_fence_before();
          __syncwarp();
          if (threadIdx.x == 0) BSA_BTRACE_AT(gc, 2 + h);
          if (lane == 0) mbar_arrive(PREADY(h));
        }
        }
        ++gc;
      }
      if (!ok) break;
      // epilogue: accA * scale -> outA, accB -> outB (rows past the tensor end
      // skipped); the two warps of a lane quarter take half of the D columns each
      const int nrows = kDKV ? p.nk : p.nq;
      const long long orow_off =
          (static_cast<long long>(it.b) * nrows + grow) * p.out_stride + static_cast<long long>(it.h) * D;
      __nv_bfloat16* rowA = p.outA + orow_off;
      __nv_bfloat16* rowB = T::kFused ? p.outB + orow_off : nullptr;
      if (it.n > 0) {
        ok = mbar_wait(DONE, dph, abort_flag, p.status, p.timeout_ns);
        if (!ok) break;
        dph ^= 1u;
        tc_fence_after();
      }
#pragma unroll 1
      for (int pass = 0; pass < (T::kFused ? 2 : 1); ++pass) {
        const uint32_t tacc = pass == 0 ? tA : tB;
        __nv_bfloat16* dst_row = pass == 0 ? rowA : rowB;
        // dK and dQ carry the softmax scale (S = scale * Q K^T); dV does not
        const float mul = (pass == 0 && kPass != kPassDV) ? p.scale : 1.0f;
#pragma unroll 1
        for (int c0 = cg * (D / 2); c0 < (cg + 1) * (D / 2); c0 += 32) {
          uint32_t ov[32];
          if (it.n > 0) {
            tmem_ld32x32b_x32(tacc + c0, ov);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = 0u;
          }
          if (grow < nrows) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(ov[2 * i]) * mul,
                                                        __uint_as_float(ov[2 * i + 1]) * mul);
              pk[i] = *reinterpret_cast<uint32_t*>(&h2);
            }
            uint4* d4 = reinterpret_cast<uint4*>(dst_row + c0);
            d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            d4[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
            d4[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
          }
        }
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kBwdMmaWarp) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
  }
}

// LSE * log2(e) and rowsum(dO * O) per (b, h, row), padded to whole 128-row tiles:
// rows past nq (and rows whose LSE is -inf, i.e. no kept key) get +inf / 0 so
// their recomputed probabilities are exactly 0.
__global__ void bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                const __nv_bfloat16* __restrict__ dout,
                                const float* __restrict__ lse, int B, int H, int nq, int D,
                                long long o_stride, int rows_pad, float* __restrict__ lse2,
                                float* __restrict__ dvec) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long total = static_cast<long long>(B) * H * rows_pad;
  if (idx >= total) return;
  const int i = static_cast<int>(idx % rows_pad);
  const long long bh = idx / rows_pad;
  const int h = static_cast<int>(bh % H), b = static_cast<int>(bh / H);
  if (i >= nq) {
    lse2[idx] = INFINITY;
    dvec[idx] = 0.f;
    return;
  }
  const float l = lse[bh * nq + i];
  lse2[idx] = l == -INFINITY ? INFINITY : l * 1.4426950408889634f;
  const long long off = (static_cast<long long>(b) * nq + i) * o_stride + static_cast<long long>(h) * D;
  const uint4* po = reinterpret_cast<const uint4*>(o + off);
  const uint4* pd = reinterpret_cast<const uint4*>(dout + off);
  float acc = 0.f;
  for (int c = 0; c < D / 8; ++c) {
    const uint4 a = __ldg(po + c), g = __ldg(pd + c);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fa = __bfloat1622float2(a2[e]), fg = __bfloat1622float2(g2[e]);
      acc = fmaf(fa.x, fg.x, acc);
      acc = fmaf(fa.y, fg.y, acc);
    }
  }
  dvec[idx] = acc;
}

// Transposed kept lists.  Pass 1: every q-tile ORs its entries, with the quadrant
// bits transposed (bit q_half*2 + k_half -> k_half*2 + q_half), into a dense
// nibble map [mask head][k-tile][q-tile].  Pass 2: one CTA per (mask head, k-tile)
// compacts its map row into an ascending list of q-tiles.
__global__ void tmap_kernel(const int* __restrict__ row_ptr, const int* __restrict__ cnt,
                            const uint32_t* __restrict__ entries, int QT, int KT, int LR, int QB,
                            int block_q, int expand, int list_heads,
                            uint32_t* __restrict__ map) {
  const int g = blockIdx.x;  // mask head * QT + q-tile
  const int mh = g / QT, qt = g - mh * QT;
  if (mh >= list_heads) return;
  const int lr = block_q >= 128 ? (qt * kBM) / block_q : qt;
  const int first_qb = block_q >= 128 ? lr : 2 * lr;
  const int n = cnt[mh * LR + lr];
  const uint32_t* ent = entries + static_cast<long long>(row_ptr[mh * QB + first_qb]) * expand;
  const int words = (QT + 7) / 8;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const uint32_t e = ent[j];
    const int kt = static_cast<int>(e & 0x0FFFFFFFu);
    const uint32_t b = e >> 28;
    const uint32_t tb = (b & 1u) | ((b >> 1) & 1u) << 2 | ((b >> 2) & 1u) << 1 | ((b >> 3) & 1u) << 3;
    atomicOr(&map[(static_cast<long long>(mh) * KT + kt) * words + (qt >> 3)], tb << (4 * (qt & 7)));
  }
}

__global__ void __launch_bounds__(256) tcompact_kernel(const uint32_t* __restrict__ map, int QT,
                                                       int KT, int* __restrict__ tcnt,
                                                       uint32_t* __restrict__ tentries) {
  __shared__ int warp_sums[8];
  const long long g = blockIdx.x;  // mask head * KT + k-tile
  const int words = (QT + 7) / 8;
  const uint32_t* row = map + g * words;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (words + 255) / 256;
  const int w0 = min(words, tid * per), w1 = min(words, w0 + per);
  int mine = 0;
  for (int w = w0; w < w1; ++w) {
    const uint32_t q = row[w];
    for (int j = 0; j < 8; ++j) mine += ((q >> (4 * j)) & 0xFu) != 0u;
  }
  int incl = mine;
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_sums[w];
  int pos = base + incl - mine;
  uint32_t* out = tentries + g * QT;
  for (int w = w0; w < w1; ++w) {
    const uint32_t q = row[w];
    for (int j = 0; j < 8; ++j) {
      const uint32_t bits = (q >> (4 * j)) & 0xFu;
      if (bits) out[pos++] = static_cast<uint32_t>(w * 8 + j) | (bits << 28);
    }
  }
  if (tid == 255) tcnt[g] = pos;
}

struct BwdGeometry {
  Geometry fwd;
  int KT;
  size_t tcnt_off, tent_off, map_off, lse_off, dvec_off, total;
};

BwdGeometry bwd_geometry(int batch, int heads, int nq, int nk, int block_q, int block_k,
                         int list_heads) {
  BwdGeometry g;
  g.fwd = geometry(batch, heads, nq, nk, block_q, block_k, list_heads);
  g.KT = ceil_div(nk, kBN);
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t mhk = static_cast<size_t>(list_heads) * g.KT;
  g.tcnt_off = up(g.fwd.total);
  g.tent_off = up(g.tcnt_off + sizeof(int) * mhk);
  g.map_off = up(g.tent_off + sizeof(uint32_t) * mhk * g.fwd.QT);
  g.lse_off = up(g.map_off + sizeof(uint32_t) * mhk * ((g.fwd.QT + 7) / 8));
  const size_t vec = sizeof(float) * static_cast<size_t>(batch) * heads * g.fwd.QT * kBM;
  g.dvec_off = up(g.lse_off + vec);
  g.total = g.dvec_off + vec;
  return g;
}

template <int D, int kPass>
int launch_bwd(const CUtensorMap& ra, const CUtensorMap& rb, const CUtensorMap& ca,
               const CUtensorMap& cb, const BwdParams& p, cudaStream_t st) {
  using C = BwdCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_kernel<D, kPass>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return record_cuda_error(e);
  int grid = device_sm_count();
  if (grid > p.total_items) grid = p.total_items;
  if (grid < 1) grid = 1;
  attn_bwd_kernel<D, kPass><<<grid, kBwdThreads, C::SMEM, st>>>(ra, rb, ca, cb, p);
  return check_launch();
}

template <int kPass>
int launch_bwd_d(int head_dim, const CUtensorMap& ra, const CUtensorMap& rb,
                 const CUtensorMap& ca, const CUtensorMap& cb, const BwdParams& p,
                 cudaStream_t st) {
  return head_dim == 128 ? launch_bwd<128, kPass>(ra, rb, ca, cb, p, st)
                         : launch_bwd<64, kPass>(ra, rb, ca, cb, p, st);
}

// BSA_BWD_SPLIT=1: three decoupled passes (dV, dK, dQ) instead of the fused dK/dV
// pass and the decoupled dQ pass.
#ifndef BSA_BWD_SPLIT
#define BSA_BWD_SPLIT 0
#endif

}  // namespace
}  // namespace bsa

extern "C" size_t bsa_attn_bwd_workspace_size(int batch, int heads, int nq, int nk, int block_q,
                                              int block_k, int list_heads) {
  if (batch < 1 || heads < 1 || nq < 1 || nk < 1 || !bsa::block_ok(block_q) ||
      !bsa::block_ok(block_k) || list_heads < 1)
    return 0;
  return bsa::bwd_geometry(batch, heads, nq, nk, block_q, block_k, list_heads).total;
}

extern "C" int bsa_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, int batch, int heads, int nq,
                            int nk, int head_dim, int qkv_row_stride, int o_row_stride,
                            int block_q, int block_k, const int* row_ptr, const int* col_idx,
                            int list_heads, float scale, void* dq, void* dk, void* dv, void* ws,
                            size_t ws_bytes, void* stream) {
  BSA_NVTX_RANGE("bsa_attn_bwd");
  using namespace bsa;
  if (!q || !k || !v || !o || !dout || !lse || !row_ptr || !col_idx || !dq || !dk || !dv || !ws)
    return BSA_ERR_INVALID_ARG;
  if (batch < 1 || heads < 1 || nq < 1 || nk < 1) return BSA_ERR_INVALID_ARG;
  if (list_heads != 1 && list_heads != batch * heads) return BSA_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, dout, static_cast<const void*>(dq),
                          static_cast<const void*>(dk), static_cast<const void*>(dv),
                          static_cast<const void*>(ws)})
    if (!aligned16(ptr)) return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  const long long qkv_rs = token_row_stride(qkv_row_stride, heads, head_dim);
  const long long o_rs = token_row_stride(o_row_stride, heads, head_dim);
  if (qkv_rs < 0 || o_rs < 0) return BSA_ERR_INVALID_ARG;
  if (!block_ok(block_q) || !block_ok(block_k)) return BSA_ERR_UNSUPPORTED;
  const BwdGeometry g = bwd_geometry(batch, heads, nq, nk, block_q, block_k, list_heads);
  if (ws_bytes < g.total) return BSA_ERR_WORKSPACE;
  if (g.fwd.nnz_cap > 0x7fffffffLL || static_cast<long long>(g.KT) >= (1LL << 28) ||
      static_cast<long long>(batch) * heads * (g.fwd.QT > g.KT ? g.fwd.QT : g.KT) > 0x3fffffffLL)
    return BSA_ERR_UNSUPPORTED;
  if (scale <= 0.0f) scale = 1.0f / sqrtf(static_cast<float>(head_dim));
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  CUtensorMap mq, mk, mv, mdo;
  if (make_map(&mq, q, batch, nq, heads, head_dim, qkv_rs) != BSA_OK ||
      make_map(&mk, k, batch, nk, heads, head_dim, qkv_rs) != BSA_OK ||
      make_map(&mv, v, batch, nk, heads, head_dim, qkv_rs) != BSA_OK ||
      make_map(&mdo, dout, batch, nq, heads, head_dim, o_rs) != BSA_OK)
    return BSA_ERR_CUDA;

  char* wsb = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(wsb);
  int* cnt = reinterpret_cast<int*>(wsb + g.fwd.cnt_off);
  uint32_t* entries = reinterpret_cast<uint32_t*>(wsb + g.fwd.ent_off);
  int* tcnt = reinterpret_cast<int*>(wsb + g.tcnt_off);
  uint32_t* tentries = reinterpret_cast<uint32_t*>(wsb + g.tent_off);
  uint32_t* map = reinterpret_cast<uint32_t*>(wsb + g.map_off);
  float* lse2 = reinterpret_cast<float*>(wsb + g.lse_off);
  float* dvec = reinterpret_cast<float*>(wsb + g.dvec_off);

  // status word + unit counters of the passes
  cudaError_t e = cudaMemsetAsync(status, 0, 4 * sizeof(int), st);  // status + 3 unit counters
  if (e == cudaSuccess) e = cudaMemsetAsync(map, 0, g.lse_off - g.map_off, st);
  if (e != cudaSuccess) return record_cuda_error(e);
  int rc = launch_build_lists(row_ptr, col_idx, list_heads, g.fwd, nk, block_q, block_k, cnt,
                              entries, status, st);
  if (rc != BSA_OK) return rc;
  const int rows_pad = g.fwd.QT * kBM;
  const long long prep_total = static_cast<long long>(batch) * heads * rows_pad;
  bwd_prep_kernel<<<static_cast<int>(ceil_div<long long>(prep_total, 256)), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, batch,
      heads, nq, head_dim, o_rs, rows_pad, lse2, dvec);
  if ((rc = check_launch()) != BSA_OK) return rc;
  tmap_kernel<<<list_heads * g.fwd.QT, 128, 0, st>>>(row_ptr, cnt, entries, g.fwd.QT, g.KT,
                                                     g.fwd.LR, g.fwd.QB, block_q, g.fwd.expand,
                                                     list_heads, map);
  if ((rc = check_launch()) != BSA_OK) return rc;
  tcompact_kernel<<<list_heads * g.KT, 256, 0, st>>>(map, g.fwd.QT, g.KT, tcnt, tentries);
  if ((rc = check_launch()) != BSA_OK) return rc;

  BwdParams p;
  p.B = batch;
  p.H = heads;
  p.nq = nq;
  p.nk = nk;
  p.QT = g.fwd.QT;
  p.KT = g.KT;
  p.list_heads = list_heads;
  p.LR = g.fwd.LR;
  p.QB = g.fwd.QB;
  p.expand = g.fwd.expand;
  p.block_q = block_q;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.row_ptr = row_ptr;
  p.cnt = cnt;
  p.entries = entries;
  p.tcnt = tcnt;
  p.tentries = tentries;
  p.lse2 = lse2;
  p.dvec = dvec;
  p.out_stride = qkv_rs;
  p.status = status;
  p.timeout_ns = 2000000000ULL;
  // key-row passes (rows = key tiles, columns = q-tiles)
  p.total_items = batch * heads * g.KT;
  if (BSA_BWD_SPLIT) {
    p.outA = static_cast<__nv_bfloat16*>(dv);
    p.outB = nullptr;
    p.unit_counter = status + 1;
    rc = launch_bwd_d<kPassDV>(head_dim, mk, mv, mq, mdo, p, st);
    if (rc != BSA_OK) return rc;
    p.outA = static_cast<__nv_bfloat16*>(dk);
    p.unit_counter = status + 3;
    rc = launch_bwd_d<kPassDK>(head_dim, mk, mv, mq, mdo, p, st);
  } else {
    p.outA = static_cast<__nv_bfloat16*>(dk);
    p.outB = static_cast<__nv_bfloat16*>(dv);
    p.unit_counter = status + 1;
    rc = launch_bwd_d<kPassDKV>(head_dim, mk, mv, mq, mdo, p, st);
  }
  if (rc != BSA_OK) return rc;
  // dQ pass (rows = q-tiles, columns = key tiles)
  p.total_items = batch * heads * g.fwd.QT;
  p.outA = static_cast<__nv_bfloat16*>(dq);
  p.outB = nullptr;
  p.unit_counter = status + 2;
  return launch_bwd_d<kPassDQ>(head_dim, mq, mdo, mk, mv, p, st);
}

#ifdef BSA_TRACE
extern "C" int bsa_btrace_dump(unsigned long long* host, size_t bytes) {
  if (bytes > sizeof(bsa::g_bsa_btrace)) bytes = sizeof(bsa::g_bsa_btrace);
  return cudaMemcpyFromSymbol(host, bsa::g_bsa_btrace, bytes) == cudaSuccess ? 0 : 4;
}
#endif
