// 3D tile permute / untile of token rows.
//
// Source: "Fast Video Generation with Sliding Tile Attention" explainer
// (aibr.jp/archives/60739), section 3 -- the latent video is a 3D token grid and
// the attention works tile by tile, so each tile's tokens are made contiguous.
//
// The permutation is closed-form: token (t, h, w) of tile (a, b, c) lands at
//   a*tT*H*W                      (all complete frame slabs before tile row a)
// + lt*b*tH*W                     (row slabs of this frame slab before b)
// + lt*lh*c*tW                    (tiles of this row slab before c)
// + ((t-a*tT)*lh + (h-b*tH))*lw + (w-c*tW)   (raster inside the tile)
// where lt, lh, lw are the (possibly ragged) extents of the tile.  The copy is a
// pure HBM stream: one warp per token row, 16-byte vector loads and stores,
// four vectors in flight per lane.
#include "bsa_common.cuh"

namespace bsa {
namespace {

struct PermGeo {
  int T, H, W, tT, tH, tW;
};

__device__ __forceinline__ long long tile_position(int tok, const PermGeo& g) {
  const int hw = g.H * g.W;
  const int t = tok / hw;
  const int rem = tok - t * hw;
  const int h = rem / g.W;
  const int w = rem - h * g.W;
  const int a = t / g.tT, b = h / g.tH, c = w / g.tW;
  const int lt = min(g.tT, g.T - a * g.tT);
  const int lh = min(g.tH, g.H - b * g.tH);
  const int lw = min(g.tW, g.W - c * g.tW);
  return static_cast<long long>(a) * g.tT * hw + static_cast<long long>(lt) * b * g.tH * g.W +
         static_cast<long long>(lt) * lh * c * g.tW +
         static_cast<long long>((t - a * g.tT) * lh + (h - b * g.tH)) * lw + (w - c * g.tW);
}

__device__ __forceinline__ void copy_row(const uint4* __restrict__ in, uint4* __restrict__ out,
                                         int vpr, int lane) {
  int c = lane;
  for (; c + 96 < vpr; c += 128) {
    uint4 v0 = __ldg(in + c), v1 = __ldg(in + c + 32), v2 = __ldg(in + c + 64),
          v3 = __ldg(in + c + 96);
    out[c] = v0;
    out[c + 32] = v1;
    out[c + 64] = v2;
    out[c + 96] = v3;
  }
  for (; c < vpr; c += 32) out[c] = __ldg(in + c);
}

// kForward: x (raster, n rows) -> y (tile order, n_pad rows, zero tail)
// !kForward: y -> x
template <bool kForward>
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* __restrict__ src,
                                                           uint4* __restrict__ dst, int n,
                                                           int n_pad, int vpr, PermGeo g,
                                                           long long total_rows) {
  const int lane = threadIdx.x & 31;
  const long long warp0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const int rows_per_batch = kForward ? n_pad : n;
  for (long long r = warp0; r < total_rows; r += nwarps) {
    const long long b = r / rows_per_batch;
    const int tok = static_cast<int>(r - b * rows_per_batch);
    if (kForward) {
      if (tok >= n) {  // zero tail of the padded sequence
        uint4* out = dst + (b * n_pad + tok) * vpr;
        for (int c = lane; c < vpr; c += 32) out[c] = make_uint4(0, 0, 0, 0);
        continue;
      }
      const long long pos = tile_position(tok, g);
      copy_row(src + (b * n + tok) * vpr, dst + (b * n_pad + pos) * vpr, vpr, lane);
    } else {
      const long long pos = tile_position(tok, g);
      copy_row(src + (b * n_pad + pos) * vpr, dst + (b * n + tok) * vpr, vpr, lane);
    }
  }
}

int permute_common(bool forward, const void* src, void* dst, int batch, int T, int H, int W,
                   int tT, int tH, int tW, int row_bytes, int n_pad, void* stream) {
  if (!src || !dst) return BSA_ERR_INVALID_ARG;
  if (batch < 1 || T < 1 || H < 1 || W < 1 || tT < 1 || tH < 1 || tW < 1 || row_bytes < 16 ||
      (row_bytes % 16) != 0)
    return BSA_ERR_INVALID_ARG;
  const long long n = static_cast<long long>(T) * H * W;
  if (n > 0x7fffffffLL || n_pad < n) return BSA_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst)) return BSA_ERR_INVALID_ARG;
  const long long vpr = row_bytes / 16;
  const char* s0 = static_cast<const char*>(src);
  const char* d0 = static_cast<const char*>(dst);
  const long long src_rows = forward ? n : n_pad, dst_rows = forward ? n_pad : n;
  const long long sb = static_cast<long long>(batch) * src_rows * row_bytes;
  const long long db = static_cast<long long>(batch) * dst_rows * row_bytes;
  if (s0 < d0 + db && d0 < s0 + sb) return BSA_ERR_INVALID_ARG;  // overlapping buffers
  PermGeo g{T, H, W, tT, tH, tW};
  const long long total_rows = static_cast<long long>(batch) * (forward ? n_pad : n);
  const int threads = 256;
  long long blocks = ceil_div<long long>(total_rows, threads / 32);
  const long long cap = static_cast<long long>(device_sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (forward)
    permute_rows_kernel<true><<<static_cast<int>(blocks), threads, 0, st>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), static_cast<int>(n), n_pad,
        static_cast<int>(vpr), g, total_rows);
  else
    permute_rows_kernel<false><<<static_cast<int>(blocks), threads, 0, st>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), static_cast<int>(n), n_pad,
        static_cast<int>(vpr), g, total_rows);
  return check_launch();
}

}  // namespace
}  // namespace bsa

extern "C" int bsa_tile_permute(const void* x, void* y, int batch, int T, int H, int W, int tT,
                                int tH, int tW, int row_bytes, int n_pad, void* stream) {
  return bsa::permute_common(true, x, y, batch, T, H, W, tT, tH, tW, row_bytes, n_pad, stream);
}

extern "C" int bsa_tile_untile(const void* y, void* x, int batch, int T, int H, int W, int tT,
                               int tH, int tW, int row_bytes, int n_pad, void* stream) {
  return bsa::permute_common(false, y, x, batch, T, H, W, tT, tH, tW, row_bytes, n_pad, stream);
}
