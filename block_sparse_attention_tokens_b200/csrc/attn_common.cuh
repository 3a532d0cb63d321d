// Pieces shared by the attention forward and backward kernels: tile constants,
// TMA tensor maps over [B, N, H, D] bf16 tensors, workspace geometry and the
// builder of per-q-tile kept lists.
#pragma once

#include <cudaTypedefs.h>

#include <mutex>

#include "bsa_common.cuh"

namespace bsa {
namespace {

constexpr int kBM = 128;  // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;  // keys per K/V tile

// ---------------------------------------------------------------------------
// Per-q-tile step lists.  One list per list row (a q-block when block_q >= 128,
// a 128-row q-tile made of two 64-row q-blocks otherwise).  Entry = k-tile index
// (bits 0-27) | quadrant bits << 28, bit (q_half * 2 + k_half) set when the
// 64x64 quadrant is kept.  Lists are written at the offset the block CSR gives
// the list row's first block row (times the k expansion), which bounds their
// length without a scan.  Malformed CSR rows are reported and left empty.
// ---------------------------------------------------------------------------
constexpr int kListThreads = 256;

// One CTA per list row.  The kept blocks of the (one or two) CSR rows are OR-ed
// into a shared-memory map holding one 4-bit quadrant mask per 128-key tile
// (eight tiles per 32-bit word); a block-wide ordered compaction then writes the
// non-empty tiles in ascending order.  Dynamic shared memory: 4 * ceil(KT / 8) bytes.
__global__ void __launch_bounds__(kListThreads) build_lists_kernel(
    const int* __restrict__ row_ptr, const int* __restrict__ col_idx, int QB, int KB, int KT,
    int LR, int block_q, int block_k, int expand, long long nnz_cap, int* __restrict__ cnt,
    uint32_t* __restrict__ entries, int* status, const int* __restrict__ page_table,
    int pages_per_batch, int heads) {
  extern __shared__ uint32_t quad[];
  __shared__ int warp_sums[kListThreads / 32];
  const int g = blockIdx.x;
  const int mh = g / LR, lr = g - mh * LR;
  const int nrows = block_q >= 128 ? 1 : ((2 * lr + 1 < QB) ? 2 : 1);
  const int first_qb = block_q >= 128 ? lr : 2 * lr;
  const int* rp = row_ptr + static_cast<long long>(mh) * QB + first_qb;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // validate the CSR rows this list reads
  bool bad = false;
  for (int r = 0; r < nrows; ++r) {
    const int b0 = rp[r], b1 = rp[r + 1];
    if (b0 < 0 || b0 > b1 || b1 > nnz_cap) {
      bad = true;
      break;
    }
    for (int i = b0 + tid; i < b1; i += kListThreads) {
      const int c = col_idx[i];
      if (c < 0 || c >= KB || (i > b0 && c <= col_idx[i - 1])) bad = true;
    }
  }
  if (__syncthreads_or(bad)) {
    if (tid == 0) {
      set_status(status, BSA_ERR_INVALID_ARG);
      cnt[g] = 0;
    }
    return;
  }
  const int words = (KT + 7) / 8;
  for (int w = tid; w < words; w += kListThreads) quad[w] = 0u;
  __syncthreads();
  // paged K/V: k-tiles on evicted pages (entry -1) are not listed; mask head mh
  // belongs to batch mh / heads (a shared list implies a single batch)
  const int* pt = page_table ? page_table + static_cast<long long>(mh / heads) * pages_per_batch
                             : nullptr;
  for (int r = 0; r < nrows; ++r) {
    // q-half bits of this row: a block of >= 128 rows covers both halves
    const uint32_t qbits = block_q >= 128 ? 0x3u : (r == 0 ? 0x1u : 0x2u);
    for (int i = rp[r] + tid; i < rp[r + 1]; i += kListThreads) {
      const int kb = col_idx[i];
      if (block_k >= 128) {
        uint32_t bits = 0;
        if (qbits & 1u) bits |= 0x3u;
        if (qbits & 2u) bits |= 0xCu;
        // a last block that overhangs nk covers fewer than `expand` k-tiles
        for (int t = 0; t < expand && kb * expand + t < KT; ++t) {
          const int kt = kb * expand + t;
          if (pt && (kt >= pages_per_batch || pt[kt] < 0)) continue;
          atomicOr(&quad[kt >> 3], bits << (4 * (kt & 7)));
        }
      } else {
        const int kt = kb >> 1, kh = kb & 1;
        if (pt && (kt >= pages_per_batch || pt[kt] < 0)) continue;
        uint32_t bits = 0;
        if (qbits & 1u) bits |= 1u << kh;
        if (qbits & 2u) bits |= 1u << (2 + kh);
        atomicOr(&quad[kt >> 3], bits << (4 * (kt & 7)));
      }
    }
  }
  __syncthreads();
  // ordered compaction: thread t owns words [t*per, (t+1)*per)
  const int per = (words + kListThreads - 1) / kListThreads;
  const int w0 = min(words, tid * per), w1 = min(words, w0 + per);
  int mine = 0;
  for (int w = w0; w < w1; ++w) {
    const uint32_t q = quad[w];
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
  uint32_t* out = entries + static_cast<long long>(rp[0]) * expand;
  for (int w = w0; w < w1; ++w) {
    const uint32_t q = quad[w];
    for (int j = 0; j < 8; ++j) {
      const uint32_t bits = (q >> (4 * j)) & 0xFu;
      if (bits) out[pos++] = static_cast<uint32_t>(w * 8 + j) | (bits << 28);
    }
  }
  if (tid == kListThreads - 1) cnt[g] = pos;
}

// Kept lists with gathered key tiles (64-token key blocks): each 128-key tile is
// any two kept key blocks of the list row, so a tile carries an empty 64-key half
// only when the row keeps an odd number of blocks.  Entry: bits 0-13 the first
// block, bits 14-27 the second block + 1 (0: none), bits 28-31 the quadrant bits
// (q_half * 2 + k_half).  Blocks both q-halves keep are paired first, ascending,
// then the blocks one q-half keeps.  One CTA per list row; dynamic shared memory
// 4 * ceil(KB / 16) bytes (2 bits per key block: which q-halves keep it).
constexpr int kGatherMaxBlocks = 16382;

__global__ void __launch_bounds__(kListThreads) build_gather_lists_kernel(
    const int* __restrict__ row_ptr, const int* __restrict__ col_idx, int QB, int KB, int LR,
    int block_q, long long nnz_cap, int* __restrict__ cnt, uint32_t* __restrict__ entries,
    int* status, const int* __restrict__ page_table, int pages_per_batch, int heads) {
  extern __shared__ uint32_t qm[];
  __shared__ int sums_a[kListThreads / 32], sums_b[kListThreads / 32];
  const int g = blockIdx.x;
  const int mh = g / LR, lr = g - mh * LR;
  const int nrows = block_q >= 128 ? 1 : ((2 * lr + 1 < QB) ? 2 : 1);
  const int first_qb = block_q >= 128 ? lr : 2 * lr;
  const int* rp = row_ptr + static_cast<long long>(mh) * QB + first_qb;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  bool bad = false;
  for (int r = 0; r < nrows; ++r) {
    const int b0 = rp[r], b1 = rp[r + 1];
    if (b0 < 0 || b0 > b1 || b1 > nnz_cap) {
      bad = true;
      break;
    }
    for (int i = b0 + tid; i < b1; i += kListThreads) {
      const int c = col_idx[i];
      if (c < 0 || c >= KB || (i > b0 && c <= col_idx[i - 1])) bad = true;
    }
  }
  if (__syncthreads_or(bad)) {
    if (tid == 0) {
      set_status(status, BSA_ERR_INVALID_ARG);
      cnt[g] = 0;
    }
    return;
  }
  const int words = (KB + 15) / 16;
  for (int w = tid; w < words; w += kListThreads) qm[w] = 0u;
  __syncthreads();
  // paged K/V: blocks on evicted pages (128-token pages hold two blocks) are dropped
  const int* pt = page_table ? page_table + static_cast<long long>(mh / heads) * pages_per_batch
                             : nullptr;
  for (int r = 0; r < nrows; ++r) {
    const uint32_t qbits = block_q >= 128 ? 0x3u : (r == 0 ? 0x1u : 0x2u);
    for (int i = rp[r] + tid; i < rp[r + 1]; i += kListThreads) {
      const int kb = col_idx[i];
      if (pt && ((kb >> 1) >= pages_per_batch || pt[kb >> 1] < 0)) continue;
      atomicOr(&qm[kb >> 4], qbits << (2 * (kb & 15)));
    }
  }
  __syncthreads();
  // thread t owns words [t*per, (t+1)*per); class A = kept by both q-halves
  const int per = (words + kListThreads - 1) / kListThreads;
  const int w0 = min(words, tid * per), w1 = min(words, w0 + per);
  int na = 0, nb = 0;
  for (int w = w0; w < w1; ++w) {
    const uint32_t q = qm[w];
    for (int j = 0; j < 16; ++j) {
      const uint32_t m = (q >> (2 * j)) & 3u;
      na += m == 3u;
      nb += m == 1u || m == 2u;
    }
  }
  int ia = na, ib = nb;
  for (int o = 1; o < 32; o <<= 1) {
    const int va = __shfl_up_sync(0xffffffffu, ia, o);
    const int vb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) {
      ia += va;
      ib += vb;
    }
  }
  if (lane == 31) {
    sums_a[warp] = ia;
    sums_b[warp] = ib;
  }
  __syncthreads();
  int base_a = 0, base_b = 0, tot_a = 0, tot_b = 0;
  for (int w = 0; w < kListThreads / 32; ++w) {
    if (w < warp) {
      base_a += sums_a[w];
      base_b += sums_b[w];
    }
    tot_a += sums_a[w];
    tot_b += sums_b[w];
  }
  const int n_entries = (tot_a + tot_b + 1) / 2;
  uint32_t* out = entries + rp[0];
  for (int e = tid; e < n_entries; e += kListThreads) out[e] = 0u;
  __syncthreads();
  int pa = base_a + ia - na, pb = tot_a + base_b + ib - nb;
  for (int w = w0; w < w1; ++w) {
    const uint32_t q = qm[w];
    for (int j = 0; j < 16; ++j) {
      const uint32_t m = (q >> (2 * j)) & 3u;
      if (m == 0u) continue;
      const int pos = m == 3u ? pa++ : pb++;
      const int kb = w * 16 + j, h = pos & 1;
      const uint32_t field = h == 0 ? static_cast<uint32_t>(kb) : static_cast<uint32_t>(kb + 1) << 14;
      const uint32_t bits = ((m & 1u) << h) | (((m >> 1) & 1u) << (2 + h));
      atomicOr(&out[pos >> 1], field | (bits << 28));
    }
  }
  if (tid == 0) cnt[g] = n_entries;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 4D map over [B, N, H, D] bf16 (D contiguous), dimensions listed innermost first as
// (D, H, N, B); consecutive token rows lie row_stride elements apart (heads * D
// for a dense tensor, more for a head slice of a wider tensor or a fused QKV
// buffer) and batches N * row_stride apart.  Box 64 x 1 x box_rows x 1 =
// box_rows token rows of 128 bytes, 128-byte swizzle.  The map covers only the
// caller's own buffer (no peer memory), and every load through it is a plain
// per-CTA TMA load.
int make_map(CUtensorMap* map, const void* base, int B, int N, int H, int D, long long row_stride,
             int box_rows = kBM) {
  auto fn = get_encode_fn();
  if (!fn) return BSA_ERR_CUDA;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(row_stride) * 2,
                           static_cast<cuuint64_t>(N) * row_stride * 2};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BSA_OK : BSA_ERR_CUDA;
}

bool block_ok(int blk) { return blk == 64 || (blk >= 128 && blk % 128 == 0); }

struct Geometry {
  int QB, KB, QT, LR, expand;
  long long nnz_cap, entries_cap;
  size_t cnt_off, ent_off, total;
};

Geometry geometry(int batch, int heads, int nq, int nk, int block_q, int block_k, int list_heads) {
  Geometry g;
  g.QB = ceil_div(nq, block_q);
  g.KB = ceil_div(nk, block_k);
  g.QT = ceil_div(nq, kBM);
  g.LR = block_q >= 128 ? g.QB : g.QT;
  g.expand = block_k >= 128 ? block_k / 128 : 1;
  g.nnz_cap = static_cast<long long>(list_heads) * g.QB * g.KB;
  g.entries_cap = g.nnz_cap * g.expand;
  g.cnt_off = kStatusBytes;
  g.ent_off = g.cnt_off + ((sizeof(int) * static_cast<size_t>(list_heads) * g.LR + 255) & ~size_t(255));
  g.total = g.ent_off + sizeof(uint32_t) * static_cast<size_t>(g.entries_cap);
  (void)batch;
  (void)heads;
  return g;
}

// Launches the kept-list builder for a call's CSR (one CTA per list row).
int launch_build_lists(const int* row_ptr, const int* col_idx, int list_heads, const Geometry& g,
                       int nk, int block_q, int block_k, int* cnt, uint32_t* entries, int* status,
                       cudaStream_t st, const int* page_table = nullptr, int pages_per_batch = 0,
                       int heads = 1, bool gather_k = false) {
  const long long lists = static_cast<long long>(list_heads) * g.LR;
  if (gather_k) {
    const size_t gsmem = sizeof(uint32_t) * static_cast<size_t>((g.KB + 15) / 16);
    if (block_k != 64 || g.KB > kGatherMaxBlocks || lists > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
    build_gather_lists_kernel<<<static_cast<int>(lists), kListThreads, gsmem, st>>>(
        row_ptr, col_idx, g.QB, g.KB, g.LR, block_q, g.nnz_cap, cnt, entries, status, page_table,
        pages_per_batch, heads);
    return check_launch();
  }
  const int KT = ceil_div(nk, kBN);
  const size_t list_smem = sizeof(uint32_t) * static_cast<size_t>((KT + 7) / 8);
  if (list_smem > 200 * 1024 || lists > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
  if (list_smem > 48 * 1024) {
    cudaError_t ea = cudaFuncSetAttribute(build_lists_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(list_smem));
    if (ea != cudaSuccess) return record_cuda_error(ea);
  }
  build_lists_kernel<<<static_cast<int>(lists), kListThreads, list_smem, st>>>(
      row_ptr, col_idx, g.QB, g.KB, KT, g.LR, block_q, block_k, g.expand, g.nnz_cap, cnt,
      entries, status, page_table, pages_per_batch, heads);
  return check_launch();
}

}  // namespace
}  // namespace bsa
