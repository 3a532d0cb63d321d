// Compaction of a uint8 block mask into per-row kept-block lists (CSR).
//
// The attention kernel walks, for each query block, only the key blocks that
// are kept; this turns the [rows][KB] byte mask into row_ptr / col_idx.
// Three short passes: per-row counts (one warp per row, 16-byte loads when the
// rows are 16-byte aligned), one exclusive scan over the rows (one CTA), and the
// ordered write of the kept indices (warp ballots, 32 columns per step).
#include "bsa_common.cuh"
#include "nvtx_range.cuh"

namespace bsa {
namespace {

__device__ __forceinline__ int count_nonzero_bytes(uint32_t w) {
  return __popc(__vcmpne4(w, 0u)) >> 3;
}

__global__ void __launch_bounds__(256) compact_count_kernel(const uint8_t* __restrict__ mask,
                                                            int rows, int kb, bool vec16,
                                                            int* __restrict__ row_ptr) {
  const int lane = threadIdx.x & 31;
  const int warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int r = warp0; r < rows; r += nwarps) {
    const uint8_t* row = mask + static_cast<long long>(r) * kb;
    int cnt = 0;
    if (vec16) {
      const uint4* v = reinterpret_cast<const uint4*>(row);
      for (int c = lane; c < kb / 16; c += 32) {
        uint4 x = __ldg(v + c);
        cnt += count_nonzero_bytes(x.x) + count_nonzero_bytes(x.y) + count_nonzero_bytes(x.z) +
               count_nonzero_bytes(x.w);
      }
    } else {
      for (int c = lane; c < kb; c += 32) cnt += row[c] != 0;
    }
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) row_ptr[r + 1] = cnt;
  }
}

// Exclusive scan of row_ptr[1..rows] in place (row_ptr[0] = 0), one CTA of 1024 threads.
__global__ void __launch_bounds__(1024) compact_scan_kernel(int* __restrict__ row_ptr, int rows) {
  __shared__ int part[1024];
  const int t = threadIdx.x;
  const int per = (rows + 1023) / 1024;
  const int lo = 1 + t * per, hi = min(rows + 1, lo + per);
  int sum = 0;
  for (int i = lo; i < hi; ++i) sum += row_ptr[i];
  part[t] = sum;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {  // inclusive Hillis-Steele scan
    int v = t >= off ? part[t - off] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  int run = t > 0 ? part[t - 1] : 0;
  for (int i = lo; i < hi; ++i) {
    run += row_ptr[i];
    row_ptr[i] = run;
  }
  if (t == 0) row_ptr[0] = 0;
}

__global__ void __launch_bounds__(256) compact_fill_kernel(const uint8_t* __restrict__ mask,
                                                           int rows, int kb,
                                                           const int* __restrict__ row_ptr,
                                                           int* __restrict__ col_idx) {
  const int lane = threadIdx.x & 31;
  const int warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int r = warp0; r < rows; r += nwarps) {
    const uint8_t* row = mask + static_cast<long long>(r) * kb;
    int out = row_ptr[r];
    for (int c0 = 0; c0 < kb; c0 += 32) {
      const int c = c0 + lane;
      const bool kept = c < kb && row[c] != 0;
      const uint32_t bal = __ballot_sync(0xffffffffu, kept);
      if (kept) col_idx[out + __popc(bal & ((1u << lane) - 1u))] = c;
      out += __popc(bal);
    }
  }
}

}  // namespace
}  // namespace bsa

extern "C" int bsa_mask_compact(const uint8_t* mask, int rows, int KB, int* row_ptr,
                                int* col_idx, void* stream) {
  BSA_NVTX_RANGE("bsa_mask_compact");
  if (!mask || !row_ptr || !col_idx || rows < 1 || KB < 1) return BSA_ERR_INVALID_ARG;
  if (static_cast<long long>(rows) * KB > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool vec16 = (KB % 16) == 0 && bsa::aligned16(mask);
  int blocks = bsa::ceil_div(rows, 8);
  const int cap = bsa::device_sm_count() * 8;
  if (blocks > cap) blocks = cap;
  bsa::compact_count_kernel<<<blocks, 256, 0, st>>>(mask, rows, KB, vec16, row_ptr);
  int rc = bsa::check_launch();
  if (rc != BSA_OK) return rc;
  bsa::compact_scan_kernel<<<1, 1024, 0, st>>>(row_ptr, rows);
  rc = bsa::check_launch();
  if (rc != BSA_OK) return rc;
  bsa::compact_fill_kernel<<<blocks, 256, 0, st>>>(mask, rows, KB, row_ptr, col_idx);
  return bsa::check_launch();
}
