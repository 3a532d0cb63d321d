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
#include "nvtx_range.cuh"

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
// vpr: 16-byte vectors copied per row; svpr / dvpr: row strides of src / dst in
// 16-byte vectors (>= vpr: a row may be a slice of a wider row, e.g. some heads).
template <bool kForward>
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* __restrict__ src,
                                                           uint4* __restrict__ dst, int n,
                                                           int n_pad, int vpr, long long svpr,
                                                           long long dvpr, PermGeo g,
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
        uint4* out = dst + (b * n_pad + tok) * dvpr;
        for (int c = lane; c < vpr; c += 32) out[c] = make_uint4(0, 0, 0, 0);
        continue;
      }
      const long long pos = tile_position(tok, g);
      copy_row(src + (b * n + tok) * svpr, dst + (b * n_pad + pos) * dvpr, vpr, lane);
    } else {
      const long long pos = tile_position(tok, g);
      copy_row(src + (b * n_pad + pos) * svpr, dst + (b * n + tok) * dvpr, vpr, lane);
    }
  }
}

// Inverse of tile_position: raster token index of tile-order position p (p < N).
__device__ __forceinline__ int tile_token(long long p, const PermGeo& g) {
  const long long hw = static_cast<long long>(g.H) * g.W;
  const long long slab = static_cast<long long>(g.tT) * hw;       // full frame slab
  const int a = static_cast<int>(p / slab);
  long long rem = p - a * slab;
  const int lt = min(g.tT, g.T - a * g.tT);
  const long long rowslab = static_cast<long long>(lt) * g.tH * g.W;
  const int b = static_cast<int>(rem / rowslab);
  rem -= b * rowslab;
  const int lh = min(g.tH, g.H - b * g.tH);
  const long long tilesz = static_cast<long long>(lt) * lh * g.tW;
  const int c = static_cast<int>(rem / tilesz);
  rem -= c * tilesz;
  const int lw = min(g.tW, g.W - c * g.tW);
  const int in = static_cast<int>(rem);
  const int t = in / (lh * lw), h = (in / lw) % lh, w = in % lw;
  return ((a * g.tT + t) * g.H + (b * g.tH + h)) * g.W + (c * g.tW + w);
}

// Tile permute fused with the per-block mean of the permuted rows (the pooling
// step of the NABLA mask): one CTA per (block of `block` output rows, 1024-column
// slice, batch).  Each thread owns 8 adjacent bf16 columns, gathers its column
// slice of every row of the block (8 rows in flight), stores it in tile order and
// sums it in fp32.  Rows past N are the zero tail and are not averaged.
// pooled: [B, heads, NB, head_dim] fp32.  svpr / dvpr: row strides of src / dst in
// 16-byte vectors (>= vpr, the vectors of the heads moved).
__global__ void __launch_bounds__(128) permute_pool_kernel(
    const uint4* __restrict__ src, uint4* __restrict__ dst, int n, int n_pad, int vpr,
    long long svpr, long long dvpr, int head_dim, int heads, int block, PermGeo g,
    float* __restrict__ pooled) {
  const int blk = blockIdx.x, b = blockIdx.z;
  const int nb = n_pad / block;
  const long long p0 = static_cast<long long>(blk) * block;
  const int rows_valid =
      static_cast<int>(max(0LL, min(static_cast<long long>(block), n - p0)));
  __shared__ int src_row[1024];
  for (int r = threadIdx.x; r < block; r += blockDim.x)
    src_row[r] = (p0 + r < n) ? tile_token(p0 + r, g) : -1;
  __syncthreads();
  const uint4* sb = src + static_cast<long long>(b) * n * svpr;
  uint4* db = dst + (static_cast<long long>(b) * n_pad + p0) * dvpr;
  for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < vpr && v < (blockIdx.y + 1) * blockDim.x;
       v += blockDim.x) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int r = 0;
    for (; r + 8 <= rows_valid; r += 8) {
      uint4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = __ldg(sb + static_cast<long long>(src_row[r + u]) * svpr + v);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        db[static_cast<long long>(r + u) * dvpr + v] = x[u];
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&x[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          acc[2 * e] += f.x;
          acc[2 * e + 1] += f.y;
        }
      }
    }
    for (; r < rows_valid; ++r) {
      const uint4 x = __ldg(sb + static_cast<long long>(src_row[r]) * svpr + v);
      db[static_cast<long long>(r) * dvpr + v] = x;
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
    for (; r < block; ++r) db[static_cast<long long>(r) * dvpr + v] = make_uint4(0, 0, 0, 0);
    const float inv = rows_valid > 0 ? 1.0f / static_cast<float>(rows_valid) : 0.f;
    const int col = v * 8, h = col / head_dim, j = col - h * head_dim;
    float4* out = reinterpret_cast<float4*>(
        pooled + ((static_cast<long long>(b) * heads + h) * nb + blk) * head_dim + j);
    out[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    out[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  }
}

// Row stride in bytes: 0 selects row_bytes (dense rows); otherwise at least
// row_bytes and a multiple of 16.  Returns -1 if invalid.
long long row_stride_bytes(long long stride, long long row_bytes) {
  if (stride == 0) return row_bytes;
  if (stride < row_bytes || (stride % 16) != 0) return -1;
  return stride;
}

// Buffers [batch][rows] of rows `row_bytes` long every `stride` bytes (the last
// row ends after row_bytes) overlap?
bool spans_overlap(const void* a, long long a_rows, long long a_stride, const void* b,
                   long long b_rows, long long b_stride, long long row_bytes) {
  const char* a0 = static_cast<const char*>(a);
  const char* b0 = static_cast<const char*>(b);
  const char* a1 = a0 + (a_rows - 1) * a_stride + row_bytes;
  const char* b1 = b0 + (b_rows - 1) * b_stride + row_bytes;
  return a0 < b1 && b0 < a1;
}

int permute_common(bool forward, const void* src, void* dst, int batch, int T, int H, int W,
                   int tT, int tH, int tW, int row_bytes, int n_pad, int src_stride_bytes,
                   int dst_stride_bytes, void* stream) {
  if (!src || !dst) return BSA_ERR_INVALID_ARG;
  if (batch < 1 || T < 1 || H < 1 || W < 1 || tT < 1 || tH < 1 || tW < 1 || row_bytes < 16 ||
      (row_bytes % 16) != 0)
    return BSA_ERR_INVALID_ARG;
  const long long n = static_cast<long long>(T) * H * W;
  if (n > 0x7fffffffLL || n_pad < n) return BSA_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst)) return BSA_ERR_INVALID_ARG;
  const long long ss = row_stride_bytes(src_stride_bytes, row_bytes);
  const long long ds = row_stride_bytes(dst_stride_bytes, row_bytes);
  if (ss < 0 || ds < 0) return BSA_ERR_INVALID_ARG;
  const long long vpr = row_bytes / 16;
  const long long src_rows = forward ? n : n_pad, dst_rows = forward ? n_pad : n;
  if (spans_overlap(src, batch * src_rows, ss, dst, batch * dst_rows, ds, row_bytes))
    return BSA_ERR_INVALID_ARG;  // overlapping buffers
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
        static_cast<int>(vpr), ss / 16, ds / 16, g, total_rows);
  else
    permute_rows_kernel<false><<<static_cast<int>(blocks), threads, 0, st>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), static_cast<int>(n), n_pad,
        static_cast<int>(vpr), ss / 16, ds / 16, g, total_rows);
  return check_launch();
}

// ---------------------------------------------------------------------------
// Per-(batch, head) slicing (SPADE summary, solution parts 1 and 3): every head
// of every batch is cut with the slice shape it chose from a menu, so the token
// order differs from head to head.  One CTA per (run of output rows, head, batch)
// moves that head's head_dim columns of each row; 16-byte vectors, head_dim / 8
// threads per row, 128 / (head_dim / 8) rows per pass, four passes in flight.
// ---------------------------------------------------------------------------
constexpr int kMaxShapes = 8;
constexpr int kSchemeThreads = 128;
constexpr int kSchemeRows = 1024;   // upper bound on the rows one CTA handles

struct ShapeMenu {
  int n;
  int t[kMaxShapes][3];
};

__device__ __forceinline__ bool menu_geo(const ShapeMenu& m, int c, int T, int H, int W,
                                         PermGeo& g) {
  if (c < 0 || c >= m.n) return false;
  g = PermGeo{T, H, W, m.t[c][0], m.t[c][1], m.t[c][2]};
  return true;
}

// Forward: raster x -> per-head tile order y (zero tail), optionally with the
// per-block means of the moved rows (pooled [B, heads, n_pad / rb, head_dim]).
// A (batch, head) whose choice is outside the menu gets zero rows and zero means
// and BSA_ERR_INVALID_ARG in *status.
template <bool kPool>
__global__ void __launch_bounds__(kSchemeThreads) scheme_permute_kernel(
    const uint4* __restrict__ src, uint4* __restrict__ dst, int n, int n_pad, int rb,
    long long svpr, long long dvpr, int heads, int head_dim, int T, int H, int W,
    const ShapeMenu menu, const int* __restrict__ choice, float* __restrict__ pooled,
    int* status) {
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const long long p0 = static_cast<long long>(blk) * rb;
  const int rows_here = static_cast<int>(min(static_cast<long long>(rb), n_pad - p0));
  PermGeo g;
  const bool good = menu_geo(menu, __ldg(choice + b * heads + h), T, H, W, g);
  if (!good && threadIdx.x == 0) set_status(status, BSA_ERR_INVALID_ARG);
  const int rows_valid =
      good ? static_cast<int>(max(0LL, min(static_cast<long long>(rows_here), n - p0))) : 0;
  __shared__ int src_row[kSchemeRows];
  __shared__ float red[kSchemeThreads * 8];
  for (int r = threadIdx.x; r < rows_valid; r += kSchemeThreads) src_row[r] = tile_token(p0 + r, g);
  __syncthreads();
  const int vph = head_dim / 8;                // 16-byte vectors of one head row
  const int rp = kSchemeThreads / vph;         // rows per pass
  const int v = threadIdx.x % vph, rg = threadIdx.x / vph;
  const uint4* sb = src + static_cast<long long>(b) * n * svpr + static_cast<long long>(h) * vph + v;
  uint4* db = dst + (static_cast<long long>(b) * n_pad + p0) * dvpr + static_cast<long long>(h) * vph + v;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  auto add = [&](const uint4& x) {
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  };
  if (rg < rp) {
    int r = rg;
    for (; r + 3 * rp < rows_valid; r += 4 * rp) {
      uint4 x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) x[u] = __ldg(sb + static_cast<long long>(src_row[r + u * rp]) * svpr);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        db[static_cast<long long>(r + u * rp) * dvpr] = x[u];
        if (kPool) add(x[u]);
      }
    }
    for (; r < rows_valid; r += rp) {
      const uint4 x = __ldg(sb + static_cast<long long>(src_row[r]) * svpr);
      db[static_cast<long long>(r) * dvpr] = x;
      if (kPool) add(x);
    }
    for (; r < rows_here; r += rp) db[static_cast<long long>(r) * dvpr] = make_uint4(0, 0, 0, 0);
  }
  if constexpr (kPool) {
    if (rg < rp) {
#pragma unroll
      for (int e = 0; e < 8; ++e) red[rg * head_dim + v * 8 + e] = acc[e];
    }
    __syncthreads();
    const float inv = rows_valid > 0 ? 1.0f / static_cast<float>(rows_valid) : 0.f;
    float* out = pooled + ((static_cast<long long>(b) * heads + h) * (n_pad / rb) + blk) * head_dim;
    for (int col = threadIdx.x; col < head_dim; col += kSchemeThreads) {
      float s = 0.f;
      for (int q = 0; q < rp; ++q) s += red[q * head_dim + col];
      out[col] = s * inv;
    }
  }
}

// Inverse: tile-order y (per-head order) -> raster x.  One CTA per (run of rb
// tile-order positions < n, head, batch).  A (batch, head) with a choice outside
// the menu gets zero rows in x (same positions, read as raster rows) and
// BSA_ERR_INVALID_ARG in *status.
__global__ void __launch_bounds__(kSchemeThreads) scheme_untile_kernel(
    const uint4* __restrict__ src, uint4* __restrict__ dst, int n, int n_pad, int rb,
    long long svpr, long long dvpr, int heads, int head_dim, int T, int H, int W,
    const ShapeMenu menu, const int* __restrict__ choice, int* status) {
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const long long p0 = static_cast<long long>(blk) * rb;
  const int rows = static_cast<int>(min(static_cast<long long>(rb), n - p0));
  PermGeo g;
  const bool good = menu_geo(menu, __ldg(choice + b * heads + h), T, H, W, g);
  if (!good && threadIdx.x == 0) set_status(status, BSA_ERR_INVALID_ARG);
  __shared__ int dst_row[kSchemeRows];
  for (int r = threadIdx.x; r < rows; r += kSchemeThreads)
    dst_row[r] = good ? tile_token(p0 + r, g) : static_cast<int>(p0 + r);
  __syncthreads();
  const int vph = head_dim / 8;
  const int rp = kSchemeThreads / vph;
  const int v = threadIdx.x % vph, rg = threadIdx.x / vph;
  if (rg >= rp) return;
  const uint4* sb = src + (static_cast<long long>(b) * n_pad + p0) * svpr + static_cast<long long>(h) * vph + v;
  uint4* db = dst + static_cast<long long>(b) * n * dvpr + static_cast<long long>(h) * vph + v;
  int r = rg;
  for (; r + 3 * rp < rows; r += 4 * rp) {
    uint4 x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      x[u] = good ? __ldg(sb + static_cast<long long>(r + u * rp) * svpr) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 4; ++u) db[static_cast<long long>(dst_row[r + u * rp]) * dvpr] = x[u];
  }
  for (; r < rows; r += rp)
    db[static_cast<long long>(dst_row[r]) * dvpr] =
        good ? __ldg(sb + static_cast<long long>(r) * svpr) : make_uint4(0, 0, 0, 0);
}

// Host checks shared by the two scheme entry points; fills the menu.
int scheme_args(const void* a, const void* b, int batch, int T, int H, int W, const int* shapes,
                int n_shapes, const int* choice, int heads, int head_dim, int n_pad,
                ShapeMenu& menu) {
  if (!a || !b || !shapes || !choice) return BSA_ERR_INVALID_ARG;
  if (batch < 1 || T < 1 || H < 1 || W < 1 || heads < 1 || head_dim < 8 || (head_dim % 8) != 0)
    return BSA_ERR_INVALID_ARG;
  if (n_shapes < 1 || n_shapes > kMaxShapes) return BSA_ERR_INVALID_ARG;
  if (head_dim > 8 * kSchemeThreads) return BSA_ERR_UNSUPPORTED;
  const long long n = static_cast<long long>(T) * H * W;
  if (n > 0x7fffffffLL || n_pad < n) return BSA_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(b) || (reinterpret_cast<uintptr_t>(choice) & 3u) != 0)
    return BSA_ERR_INVALID_ARG;
  menu.n = n_shapes;
  for (int i = 0; i < kMaxShapes; ++i)
    for (int j = 0; j < 3; ++j) menu.t[i][j] = i < n_shapes ? shapes[3 * i + j] : 1;
  for (int i = 0; i < n_shapes; ++i)
    if (menu.t[i][0] < 1 || menu.t[i][1] < 1 || menu.t[i][2] < 1) return BSA_ERR_INVALID_ARG;
  return BSA_OK;
}

}  // namespace
}  // namespace bsa

extern "C" int bsa_tile_permute_pool(const void* x, void* y, int batch, int T, int H, int W,
                                     int tT, int tH, int tW, int heads, int head_dim, int n_pad,
                                     int block, float* pooled, int x_row_stride, int y_row_stride,
                                     void* stream) {
  BSA_NVTX_RANGE("bsa_tile_permute_pool");
  using namespace bsa;
  if (!x || !y || !pooled) return BSA_ERR_INVALID_ARG;
  if (batch < 1 || T < 1 || H < 1 || W < 1 || tT < 1 || tH < 1 || tW < 1 || heads < 1 ||
      head_dim < 8 || (head_dim % 8) != 0 || block < 1 || block > 1024)
    return BSA_ERR_INVALID_ARG;
  const long long n = static_cast<long long>(T) * H * W;
  if (n > 0x7fffffffLL || n_pad < n || (n_pad % block) != 0) return BSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(pooled)) return BSA_ERR_INVALID_ARG;
  const long long row_bytes = static_cast<long long>(heads) * head_dim * 2;
  const long long xs = row_stride_bytes(2LL * x_row_stride, row_bytes);
  const long long ys = row_stride_bytes(2LL * y_row_stride, row_bytes);
  if (x_row_stride < 0 || y_row_stride < 0 || xs < 0 || ys < 0) return BSA_ERR_INVALID_ARG;
  if (spans_overlap(x, batch * n, xs, y, batch * static_cast<long long>(n_pad), ys, row_bytes))
    return BSA_ERR_INVALID_ARG;
  PermGeo g{T, H, W, tT, tH, tW};
  const int vpr = static_cast<int>(row_bytes / 16);
  dim3 grid(n_pad / block, ceil_div(vpr, 128), batch);
  permute_pool_kernel<<<grid, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(x), static_cast<uint4*>(y), static_cast<int>(n), n_pad, vpr,
      xs / 16, ys / 16, head_dim, heads, block, g, pooled);
  return check_launch();
}

extern "C" int bsa_tile_permute(const void* x, void* y, int batch, int T, int H, int W, int tT,
                                int tH, int tW, int row_bytes, int n_pad, int x_row_stride_bytes,
                                int y_row_stride_bytes, void* stream) {
  BSA_NVTX_RANGE("bsa_tile_permute");
  return bsa::permute_common(true, x, y, batch, T, H, W, tT, tH, tW, row_bytes, n_pad,
                             x_row_stride_bytes, y_row_stride_bytes, stream);
}

extern "C" int bsa_tile_untile(const void* y, void* x, int batch, int T, int H, int W, int tT,
                               int tH, int tW, int row_bytes, int n_pad, int y_row_stride_bytes,
                               int x_row_stride_bytes, void* stream) {
  BSA_NVTX_RANGE("bsa_tile_untile");
  return bsa::permute_common(false, y, x, batch, T, H, W, tT, tH, tW, row_bytes, n_pad,
                             y_row_stride_bytes, x_row_stride_bytes, stream);
}

extern "C" int bsa_scheme_permute(const void* x, void* y, int batch, int T, int H, int W,
                                  const int* shapes, int n_shapes, const int* choice, int heads,
                                  int head_dim, int n_pad, int block, float* pooled,
                                  int x_row_stride, int y_row_stride, int* device_status,
                                  void* stream) {
  BSA_NVTX_RANGE("bsa_scheme_permute");
  using namespace bsa;
  ShapeMenu menu;
  const int rc = scheme_args(x, y, batch, T, H, W, shapes, n_shapes, choice, heads, head_dim,
                             n_pad, menu);
  if (rc != BSA_OK) return rc;
  if (pooled) {
    if (block < 1 || block > kSchemeRows || (n_pad % block) != 0 || !aligned16(pooled))
      return BSA_ERR_INVALID_ARG;
  } else if (block < 0 || block > kSchemeRows) {
    return BSA_ERR_INVALID_ARG;
  }
  const int rb = block > 0 ? block : 64;
  const long long n = static_cast<long long>(T) * H * W;
  const long long row_bytes = static_cast<long long>(heads) * head_dim * 2;
  const long long xs = row_stride_bytes(2LL * x_row_stride, row_bytes);
  const long long ys = row_stride_bytes(2LL * y_row_stride, row_bytes);
  if (x_row_stride < 0 || y_row_stride < 0 || xs < 0 || ys < 0) return BSA_ERR_INVALID_ARG;
  if (spans_overlap(x, batch * n, xs, y, batch * static_cast<long long>(n_pad), ys, row_bytes))
    return BSA_ERR_INVALID_ARG;
  dim3 grid(static_cast<unsigned>(ceil_div<long long>(n_pad, rb)), heads, batch);
  if (grid.y > 65535u || grid.z > 65535u) return BSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (pooled)
    scheme_permute_kernel<true><<<grid, kSchemeThreads, 0, st>>>(
        static_cast<const uint4*>(x), static_cast<uint4*>(y), static_cast<int>(n), n_pad, rb,
        xs / 16, ys / 16, heads, head_dim, T, H, W, menu, choice, pooled, device_status);
  else
    scheme_permute_kernel<false><<<grid, kSchemeThreads, 0, st>>>(
        static_cast<const uint4*>(x), static_cast<uint4*>(y), static_cast<int>(n), n_pad, rb,
        xs / 16, ys / 16, heads, head_dim, T, H, W, menu, choice, nullptr, device_status);
  return check_launch();
}

extern "C" int bsa_scheme_untile(const void* y, void* x, int batch, int T, int H, int W,
                                 const int* shapes, int n_shapes, const int* choice, int heads,
                                 int head_dim, int n_pad, int y_row_stride, int x_row_stride,
                                 int* device_status, void* stream) {
  BSA_NVTX_RANGE("bsa_scheme_untile");
  using namespace bsa;
  ShapeMenu menu;
  const int rc = scheme_args(y, x, batch, T, H, W, shapes, n_shapes, choice, heads, head_dim,
                             n_pad, menu);
  if (rc != BSA_OK) return rc;
  const long long n = static_cast<long long>(T) * H * W;
  const long long row_bytes = static_cast<long long>(heads) * head_dim * 2;
  const long long ys = row_stride_bytes(2LL * y_row_stride, row_bytes);
  const long long xs = row_stride_bytes(2LL * x_row_stride, row_bytes);
  if (x_row_stride < 0 || y_row_stride < 0 || xs < 0 || ys < 0) return BSA_ERR_INVALID_ARG;
  if (spans_overlap(y, batch * static_cast<long long>(n_pad), ys, x, batch * n, xs, row_bytes))
    return BSA_ERR_INVALID_ARG;
  constexpr int rb = 128;
  dim3 grid(static_cast<unsigned>(ceil_div<long long>(n, rb)), heads, batch);
  if (grid.y > 65535u || grid.z > 65535u) return BSA_ERR_UNSUPPORTED;
  scheme_untile_kernel<<<grid, kSchemeThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(y), static_cast<uint4*>(x), static_cast<int>(n), n_pad, rb,
      ys / 16, xs / 16, heads, head_dim, T, H, W, menu, choice, device_status);
  return check_launch();
}
