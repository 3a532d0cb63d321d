// Static block masks: Sliding-Tile window and radial energy-decay.
//
// Sliding Tile Attention: "Fast Video Generation with Sliding Tile Attention"
// explainer (aibr.jp/archives/60739), sections 2-3 -- a query tile attends to the
// tiles inside a window counted in tiles (not tokens).
// Radial attention: "Radial Attention" explainer (aibr.jp/archives/112136),
// sections 1-3 -- dense for temporally close tokens, spatial window shrinking as
// the temporal distance grows, O(n log n) kept pairs.
//
// Both masks are pure functions of the block indices: one thread per mask byte,
// consecutive threads write consecutive bytes of a row (coalesced).
#include "bsa_common.cuh"
#include "nvtx_range.cuh"

namespace bsa {
namespace {

__device__ __forceinline__ bool sta_axis(int a, int a2, int n, int w, int shift) {
  const int lo_off = (w - 1) / 2, hi_off = w / 2;
  int lo, hi;
  if (shift) {
    int start = a - lo_off;
    start = min(start, max(n - w, 0));
    start = max(start, 0);
    lo = start;
    hi = min(start + w, n) - 1;
  } else {
    lo = max(a - lo_off, 0);
    hi = min(a + hi_off, n - 1);
  }
  return a2 >= lo && a2 <= hi;
}

__global__ void sta_mask_kernel(int nT, int nH, int nW, int wT, int wH, int wW, int shift,
                                uint8_t* __restrict__ mask, long long total) {
  const long long n = static_cast<long long>(nT) * nH * nW;
  for (long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
       idx < total; idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int q = static_cast<int>(idx / n);
    const int k = static_cast<int>(idx - static_cast<long long>(q) * n);
    const int qa = q / (nH * nW), qb = (q / nW) % nH, qc = q % nW;
    const int ka = k / (nH * nW), kb = (k / nW) % nH, kc = k % nW;
    const bool keep = sta_axis(qa, ka, nT, wT, shift) && sta_axis(qb, kb, nH, wH, shift) &&
                      sta_axis(qc, kc, nW, wW, shift);
    mask[idx] = keep ? 1 : 0;
  }
}

// Window of frame distance `dist` >= 2: keep iff frame_kept && 2*gap*den < num.
__device__ __forceinline__ void radial_params(long long dist, long long S, long long B,
                                              bool& frame_kept, long long& num,
                                              long long& den) {
  const int r = 63 - __clzll(dist);  // floor(log2 dist)
  if (S >= (B << r)) {
    frame_kept = true;
    num = S;
    den = 1LL << r;
    return;
  }
  int c = 0;
  while ((S << c) < (B << r)) ++c;
  frame_kept = (dist & ((1LL << c) - 1)) == 0;
  num = B;
  den = 1;
}

__global__ void radial_mask_kernel(long long n_tokens, long long S, long long B, int nb,
                                   uint8_t* __restrict__ mask, long long total) {
  for (long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
       idx < total; idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long qb = idx / nb, kb = idx - qb * nb;
    const long long q_lo = qb * B, q_hi = min(q_lo + B, n_tokens);  // [lo, hi)
    const long long k_lo = kb * B, k_hi = min(k_lo + B, n_tokens);
    bool keep = false;
    // walk the per-frame pieces of both blocks
    for (long long qs = q_lo; qs < q_hi && !keep;) {
      const long long fq = qs / S;
      const long long qe = min(q_hi, (fq + 1) * S);
      const long long a0 = qs - fq * S, a1 = qe - 1 - fq * S;
      for (long long ks = k_lo; ks < k_hi;) {
        const long long fk = ks / S;
        const long long ke = min(k_hi, (fk + 1) * S);
        const long long b0 = ks - fk * S, b1 = ke - 1 - fk * S;
        const long long dist = fq > fk ? fq - fk : fk - fq;
        if (dist <= 1) {
          keep = true;
          break;
        }
        bool frame_kept;
        long long num, den;
        radial_params(dist, S, B, frame_kept, num, den);
        long long gap = b0 - a1;
        if (a0 - b1 > gap) gap = a0 - b1;
        if (gap < 0) gap = 0;
        if (frame_kept && 2 * gap * den < num) {
          keep = true;
          break;
        }
        ks = ke;
      }
      qs = qe;
    }
    mask[idx] = keep ? 1 : 0;
  }
}

int grid_for(long long total, int threads) {
  long long blocks = ceil_div<long long>(total, threads);
  const long long cap = static_cast<long long>(device_sm_count()) * 16;
  return static_cast<int>(blocks < cap ? (blocks < 1 ? 1 : blocks) : cap);
}

}  // namespace
}  // namespace bsa

extern "C" int bsa_sta_mask(int nT, int nH, int nW, int wT, int wH, int wW, int shift,
                            uint8_t* mask, void* stream) {
  BSA_NVTX_RANGE("bsa_sta_mask");
  if (!mask || nT < 1 || nH < 1 || nW < 1 || wT < 1 || wH < 1 || wW < 1) return BSA_ERR_INVALID_ARG;
  const long long n = static_cast<long long>(nT) * nH * nW;
  if (n > (1LL << 20)) return BSA_ERR_UNSUPPORTED;
  const long long total = n * n;
  bsa::sta_mask_kernel<<<bsa::grid_for(total, 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      nT, nH, nW, wT, wH, wW, shift ? 1 : 0, mask, total);
  return bsa::check_launch();
}

extern "C" int bsa_radial_mask(int n_tokens, int tokens_per_frame, int block, uint8_t* mask,
                               void* stream) {
  BSA_NVTX_RANGE("bsa_radial_mask");
  if (!mask || n_tokens < 1 || tokens_per_frame < 1 || block < 1) return BSA_ERR_INVALID_ARG;
  const long long nb = bsa::ceil_div<long long>(n_tokens, block);
  if (nb > (1LL << 20)) return BSA_ERR_UNSUPPORTED;
  const long long total = nb * nb;
  bsa::radial_mask_kernel<<<bsa::grid_for(total, 256), 256, 0,
                            static_cast<cudaStream_t>(stream)>>>(
      n_tokens, tokens_per_frame, block, static_cast<int>(nb), mask, total);
  return bsa::check_launch();
}
