// SPADE scheme generation on sm_100a: SICS of every block of a slicing and the
// per-head choice of a slicing from a menu of 3D block shapes.
//
// Source: the SPADE summary (gist.science/ja/paper/2608.03335), solution part 1
// (a menu of ways to slice the T x H x W token grid: wide and flat, tall and thin,
// mixed) and part 2 (scheme generation: SICS, the sum of intra-block cosine
// similarities, decided per head from Q and K alone at a small fraction of the
// attention time).
//
// SICS(block) = sum over ordered token pairs (i, j) of the block of cos(x_i, x_j)
//             = || sum_i x_i / |x_i| ||^2,
// so one pass over the block's tokens suffices: every token vector is normalised
// and added to a per-head fp32 sum whose squared norm is the block's SICS.  The
// kernel is HBM-bound: each token row (heads x head_dim bf16) is read once per
// slicing.
#include "bsa_common.cuh"
#include "nvtx_range.cuh"

#include <cuda_bf16.h>

namespace bsa {
namespace {

constexpr int kMaxShapes = 16;
constexpr int kMaxTileTokens = 4096;

struct SicsGrid {
  int T, H, W, tT, tH, tW, nT, nH, nW;
};

SicsGrid sics_grid(int T, int H, int W, int tT, int tH, int tW) {
  SicsGrid g{T, H, W, tT, tH, tW, ceil_div(T, tT), ceil_div(H, tH), ceil_div(W, tW)};
  return g;
}

// A launch covers up to 2 * kMaxShapes segments (a tensor under one slicing); the
// CTAs of segment s are blockIdx.x in [first[s], first[s + 1]), one per tile.
struct SicsSegments {
  int n;
  long long row_vec;  // token row stride in 16-byte vectors (>= heads * head_dim / 8)
  int first[2 * kMaxShapes + 1];
  SicsGrid g[2 * kMaxShapes];
  const uint4* x[2 * kMaxShapes];
  float* out[2 * kMaxShapes];  // [batch][heads][tiles of the segment]
};

// One CTA per (segment tile, batch).  Thread j owns the 8 bf16 at [8j, 8j + 8) of
// a token row; the G = D / 8 consecutive threads of one head reduce that head's
// squared norm with shuffles.  Four token rows are loaded per iteration.
template <int D>
__global__ void __launch_bounds__(1024) sics_kernel(const __grid_constant__ SicsSegments sg,
                                                   int heads) {
  constexpr int G = D / 8;
  __shared__ long long tok_off[kMaxTileTokens];
  int seg = 0;
  while (seg + 1 < sg.n && static_cast<int>(blockIdx.x) >= sg.first[seg + 1]) ++seg;
  const SicsGrid& g = sg.g[seg];
  const uint4* __restrict__ x = sg.x[seg];
  const int tile = blockIdx.x - sg.first[seg], b = blockIdx.y;
  const long long row_vec = sg.row_vec;   // 16-byte vectors from one token row to the next
  const int j = threadIdx.x;
  const bool active = j < heads * G;
  const int a = tile / (g.nH * g.nW);
  const int rem = tile - a * (g.nH * g.nW);
  const int bb = rem / g.nW, c = rem - bb * g.nW;
  const int t0 = a * g.tT, h0 = bb * g.tH, w0 = c * g.tW;
  const int vT = min(g.tT, g.T - t0), vH = min(g.tH, g.H - h0), vW = min(g.tW, g.W - w0);
  const int n = vT * vH * vW;
  const long long n_tok = static_cast<long long>(g.T) * g.H * g.W;
  for (int r = j; r < n; r += blockDim.x) {
    const int dt = r / (vH * vW), rest = r - dt * (vH * vW);
    const int dh = rest / vW, dw = rest - dh * vW;
    const long long tok = (static_cast<long long>(t0 + dt) * g.H + (h0 + dh)) * g.W + (w0 + dw);
    tok_off[r] = (static_cast<long long>(b) * n_tok + tok) * row_vec;
  }
  __syncthreads();
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int r0 = 0; r0 < n; r0 += 4) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (active && r0 + u < n) v[u] = __ldg(x + tok_off[r0 + u] + j);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
      float f[8];
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 p = __bfloat1622float2(h2[e]);
        f[2 * e] = p.x;
        f[2 * e + 1] = p.y;
        ss = fmaf(p.x, p.x, ss);
        ss = fmaf(p.y, p.y, ss);
      }
#pragma unroll
      for (int o = G / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      // a zero vector has no direction and adds nothing
      const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(f[e], inv, acc[e]);
    }
  }
  float part = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) part = fmaf(acc[e], acc[e], part);
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if (active && (j % G) == 0) {
    const int h = j / G;
    const int ntiles = g.nT * g.nH * g.nW;
    sg.out[seg][(static_cast<long long>(b) * heads + h) * ntiles + tile] = part;
  }
}

struct SicsMenu {
  int n;
  int ntiles[kMaxShapes];
  long long off[kMaxShapes];   // float offset of the shape's [B][heads][ntiles] block (Q)
  float inv_pairs[kMaxShapes]; // 1 / (2 * sum over tiles of n_b^2)
};

// One CTA per (batch, head): each shape's score is the sum of the Q and K block
// SICS over all tiles times inv_pairs; the choice is the first maximum.
__global__ void __launch_bounds__(256) sics_scheme_kernel(const float* __restrict__ sq,
                                                          const float* __restrict__ sk,
                                                          SicsMenu m, int BH,
                                                          float* __restrict__ scores,
                                                          int* __restrict__ choice) {
  __shared__ float warp_part[8];
  __shared__ float sc[kMaxShapes];
  const int bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int s = 0; s < m.n; ++s) {
    const long long base = m.off[s] + static_cast<long long>(bh) * m.ntiles[s];
    float v = 0.f;
    for (int t = tid; t < m.ntiles[s]; t += 256) v += sq[base + t] + sk[base + t];
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) warp_part[warp] = v;
    __syncthreads();
    if (tid == 0) {
      float tot = 0.f;
      for (int w = 0; w < 8; ++w) tot += warp_part[w];
      sc[s] = tot * m.inv_pairs[s];
    }
    __syncthreads();
  }
  if (tid == 0) {
    int best = 0;
    for (int s = 0; s < m.n; ++s) {
      scores[static_cast<long long>(bh) * m.n + s] = sc[s];
      if (sc[s] > sc[best]) best = s;
    }
    choice[bh] = best;
  }
  (void)BH;
}

int check_sics_args(int batch, int T, int H, int W, int heads, int head_dim) {
  if (batch < 1 || T < 1 || H < 1 || W < 1 || heads < 1) return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (heads * (head_dim / 8) > 1024 || batch > 65535) return BSA_ERR_UNSUPPORTED;
  return BSA_OK;
}

int check_shape(int T, int H, int W, int tT, int tH, int tW) {
  // a tile may exceed the grid along an axis: it is then one ragged tile there
  if (tT < 1 || tH < 1 || tW < 1) return BSA_ERR_INVALID_ARG;
  if (static_cast<long long>(tT) * tH * tW > kMaxTileTokens) return BSA_ERR_UNSUPPORTED;
  const long long nt = static_cast<long long>(ceil_div(T, tT)) * ceil_div(H, tH) * ceil_div(W, tW);
  if (nt > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
  return BSA_OK;
}

int launch_sics(const SicsSegments& sg, int batch, int heads, int head_dim, cudaStream_t st) {
  const int threads = ((heads * (head_dim / 8) + 31) / 32) * 32;
  dim3 grid(sg.first[sg.n], batch);
  if (head_dim == 128)
    sics_kernel<128><<<grid, threads, 0, st>>>(sg, heads);
  else
    sics_kernel<64><<<grid, threads, 0, st>>>(sg, heads);
  return check_launch();
}

// sum over tiles of n_b^2 factorises over the three axes
double pairs_of(int T, int H, int W, int tT, int tH, int tW) {
  auto axis = [](int n, int t) {
    double s = 0.0;
    for (int a = 0; a < n; a += t) {
      const double v = static_cast<double>(n - a < t ? n - a : t);
      s += v * v;
    }
    return s;
  };
  return axis(T, tT) * axis(H, tH) * axis(W, tW);
}

}  // namespace
}  // namespace bsa

extern "C" int bsa_sics_blocks(const void* x, int batch, int T, int H, int W, int tT, int tH,
                               int tW, int heads, int head_dim, int row_stride, float* out,
                               void* stream) {
  BSA_NVTX_RANGE("bsa_sics_blocks");
  using namespace bsa;
  if (!x || !out || !aligned16(x)) return BSA_ERR_INVALID_ARG;
  int rc = check_sics_args(batch, T, H, W, heads, head_dim);
  if (rc != BSA_OK) return rc;
  if ((rc = check_shape(T, H, W, tT, tH, tW)) != BSA_OK) return rc;
  const long long rs = token_row_stride(row_stride, heads, head_dim);
  if (rs < 0) return BSA_ERR_INVALID_ARG;
  SicsSegments sg;
  sg.row_vec = rs / 8;
  sg.n = 1;
  sg.g[0] = sics_grid(T, H, W, tT, tH, tW);
  sg.x[0] = static_cast<const uint4*>(x);
  sg.out[0] = out;
  sg.first[0] = 0;
  sg.first[1] = sg.g[0].nT * sg.g[0].nH * sg.g[0].nW;
  return launch_sics(sg, batch, heads, head_dim, static_cast<cudaStream_t>(stream));
}

extern "C" size_t bsa_sics_workspace_size(int batch, int heads, int T, int H, int W,
                                          const int* shapes, int n_shapes) {
  using namespace bsa;
  if (!shapes || n_shapes < 1 || n_shapes > kMaxShapes || batch < 1 || heads < 1) return 0;
  size_t floats = 0;
  for (int s = 0; s < n_shapes; ++s) {
    const int* sh = shapes + 3 * s;
    if (check_shape(T, H, W, sh[0], sh[1], sh[2]) != BSA_OK) return 0;
    floats += 2ull * batch * heads * ceil_div(T, sh[0]) * ceil_div(H, sh[1]) * ceil_div(W, sh[2]);
  }
  return floats * sizeof(float);
}

extern "C" int bsa_sics_scheme(const void* q, const void* k, int batch, int T, int H, int W,
                               int heads, int head_dim, int row_stride, const int* shapes,
                               int n_shapes, float* scores, int* choice, void* ws,
                               size_t ws_bytes, void* stream) {
  BSA_NVTX_RANGE("bsa_sics_scheme");
  using namespace bsa;
  if (!q || !k || !shapes || !scores || !choice || !ws || !aligned16(q) || !aligned16(k))
    return BSA_ERR_INVALID_ARG;
  if (n_shapes < 1 || n_shapes > kMaxShapes) return BSA_ERR_INVALID_ARG;
  int rc = check_sics_args(batch, T, H, W, heads, head_dim);
  if (rc != BSA_OK) return rc;
  for (int s = 0; s < n_shapes; ++s)
    if ((rc = check_shape(T, H, W, shapes[3 * s], shapes[3 * s + 1], shapes[3 * s + 2])) != BSA_OK)
      return rc;
  const long long rs = token_row_stride(row_stride, heads, head_dim);
  if (rs < 0) return BSA_ERR_INVALID_ARG;
  const size_t need = bsa_sics_workspace_size(batch, heads, T, H, W, shapes, n_shapes);
  if (ws_bytes < need) return BSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* wsf = static_cast<float*>(ws);
  // every (tensor, shape) pair is one segment of a single launch: Q's block SICS of
  // all shapes first, then K's
  SicsMenu m;
  m.n = n_shapes;
  SicsSegments sg;
  sg.row_vec = rs / 8;
  sg.n = 2 * n_shapes;
  long long off = 0, ctas = 0;
  for (int s = 0; s < n_shapes; ++s) {
    const SicsGrid g = sics_grid(T, H, W, shapes[3 * s], shapes[3 * s + 1], shapes[3 * s + 2]);
    const int nt = g.nT * g.nH * g.nW;
    m.ntiles[s] = nt;
    m.off[s] = off;
    m.inv_pairs[s] = static_cast<float>(
        1.0 / (2.0 * pairs_of(T, H, W, shapes[3 * s], shapes[3 * s + 1], shapes[3 * s + 2])));
    off += static_cast<long long>(batch) * heads * nt;
  }
  const long long total_q = off;
  for (int seg = 0; seg < 2 * n_shapes; ++seg) {
    const int s = seg % n_shapes;
    sg.g[seg] = sics_grid(T, H, W, shapes[3 * s], shapes[3 * s + 1], shapes[3 * s + 2]);
    sg.x[seg] = static_cast<const uint4*>(seg < n_shapes ? q : k);
    sg.out[seg] = wsf + (seg < n_shapes ? 0 : total_q) + m.off[s];
    sg.first[seg] = static_cast<int>(ctas);
    ctas += m.ntiles[s];
  }
  if (ctas > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
  sg.first[2 * n_shapes] = static_cast<int>(ctas);
  if ((rc = launch_sics(sg, batch, heads, head_dim, st)) != BSA_OK) return rc;
  sics_scheme_kernel<<<batch * heads, 256, 0, st>>>(wsf, wsf + total_q, m, batch * heads, scores,
                                                    choice);
  return check_launch();
}
