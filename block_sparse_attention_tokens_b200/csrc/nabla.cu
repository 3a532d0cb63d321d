// NABLA dynamic block mask: block mean-pooling of Q and K, then a per-row
// softmax over the pooled logits and the smallest top set reaching mass p.
//
// Source: "NABLA (Neighborhood Adaptive Block-Level Attention)" explainer
// (aibr.jp/archives/124678), section 3 -- Q and K are average-pooled per block,
// full attention is computed on the pooled tokens, each row is thresholded by its
// cumulative distribution and the binary result is applied at block level.
// Forced key ranges (anchors / recent frames): "Sparse Forcing" summary
// (gist.science/ja/paper/2604.21221), part 2.
//
// Kernels
//   pool   : HBM-bound column sums.  One CTA per (tensor, batch, block, 1024-column
//            chunk); each thread owns 8 adjacent bf16 columns (one 16-byte vector
//            per token row) and accumulates in fp32 over the block's valid rows.
//   select : one CTA per (batch, head, up to 8 query blocks: fewer when the key
//            range is long, so that the rows' logits fit in shared memory).
//            Pooled keys stream through shared memory in tiles of 32 blocks;
//            every thread forms one (partial) logit per tile.  Each warp then
//            owns one query row: softmax
//            statistics, a 32-step radix search over the order-preserving integer
//            image of the fp32 logits for the cut, ties resolved to the lower
//            block index, and the row of mask bytes.
#include "bsa_common.cuh"
#include "nvtx_range.cuh"

namespace bsa {
namespace {

constexpr int kPoolThreads = 128;          // threads per pooling CTA
constexpr int kPoolCols = kPoolThreads * 8;  // bf16 columns per pooling CTA
constexpr int kSelRows = 8;                // query rows per select CTA (one per warp)
constexpr int kSelTile = 32;               // key blocks per shared-memory tile

__device__ __forceinline__ void add_bf16x8(float* acc, const uint4& v) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(p[i]);
    acc[2 * i] += f.x;
    acc[2 * i + 1] += f.y;
  }
}

// grid: x = block index, y = column chunk, z = batch * 2 + tensor (0 = q, 1 = k)
__global__ void __launch_bounds__(kPoolThreads) nabla_pool_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, int heads,
    int head_dim, long long row_stride, int nq, int nk, int block, int qb_count, int kb_count,
    float* __restrict__ qbar, float* __restrict__ kbar) {
  const int which = blockIdx.z & 1;
  const int b = blockIdx.z >> 1;
  const int nblk = which ? kb_count : qb_count;
  const int blk = blockIdx.x;
  if (blk >= nblk) return;
  const int n = which ? nk : nq;
  const __nv_bfloat16* src = which ? k : q;
  float* dst = which ? kbar : qbar;
  const int C = heads * head_dim;
  const int col = blockIdx.y * kPoolCols + threadIdx.x * 8;
  if (col >= C) return;
  const int r0 = blk * block;
  const int r1 = min(r0 + block, n);
  const uint4* base =
      reinterpret_cast<const uint4*>(src + (static_cast<long long>(b) * n + r0) * row_stride + col);
  const long long stride = row_stride / 8;  // uint4 per token row
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  int r = r0;
  for (; r + 4 <= r1; r += 4) {
    const uint4* p = base + static_cast<long long>(r - r0) * stride;
    uint4 v0 = __ldg(p), v1 = __ldg(p + stride), v2 = __ldg(p + 2 * stride),
          v3 = __ldg(p + 3 * stride);
    add_bf16x8(acc, v0);
    add_bf16x8(acc, v1);
    add_bf16x8(acc, v2);
    add_bf16x8(acc, v3);
  }
  for (; r < r1; ++r) add_bf16x8(acc, __ldg(base + static_cast<long long>(r - r0) * stride));
  const float inv = 1.0f / static_cast<float>(r1 - r0);
  const int h = col / head_dim, j = col - h * head_dim;
  float4* out = reinterpret_cast<float4*>(
      dst + ((static_cast<long long>(b) * heads + h) * nblk + blk) * head_dim + j);
  out[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  out[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
}

__device__ __forceinline__ uint32_t order_key(float z) {
  const uint32_t u = __float_as_uint(z);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_isum(int v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The cut of one row's top-p selection: the largest order key v whose mass
// F(v) = sum of e_c over the keys >= v reaches target, found bit by bit from the
// top.  Each lane sums its entries c = lane, lane + 32, ... in that order, so the
// register form (rows of up to 512 candidates, the keys and values held by the
// lanes) and the shared-memory form give the same sums.
template <int NREG>
__device__ __forceinline__ uint32_t radix_cut_regs(const float* z, const float* e, int nr,
                                                   int lane, float target) {
  uint32_t kr[NREG];
  float er[NREG];
#pragma unroll
  for (int i = 0; i < NREG; ++i) {
    const int c = lane + 32 * i;
    kr[i] = c < nr ? order_key(z[c]) : 0u;   // 0 is below every candidate (>= 1)
    er[i] = c < nr ? e[c] : 0.f;
  }
  uint32_t v = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = v | (1u << bit);
    float f = 0.f;
#pragma unroll
    for (int i = 0; i < NREG; ++i)
      if (kr[i] >= cand) f += er[i];
    f = warp_sum(f);
    if (f >= target) v = cand;
  }
  return v;
}

__device__ __forceinline__ uint32_t radix_cut(const float* z, const float* e, int nr,
                                              int lane, float target) {
  uint32_t v = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = v | (1u << bit);
    float f = 0.f;
    for (int c = lane; c < nr; c += 32)
      if (order_key(z[c]) >= cand) f += e[c];
    f = warp_sum(f);
    if (f >= target) v = cand;
  }
  return v;
}

// grid: x = ceil(QB / rows), y = heads, z = batch; 256 threads (8 warps).
// `rows` (1, 2, 4 or 8) query rows per CTA, chosen by the host so that the rows'
// logits fit in shared memory: 8 for short key ranges, fewer for long ones.  In
// the logit phase the 8 warps split head_dim: warp w forms, for every row of the
// CTA and the 32 key blocks of a tile (one per lane), the partial dot product over
// its D / 8 columns -- the query values as 16-byte broadcast loads, the key values
// from a transposed tile -- and the partials are added in warp order.  In the
// selection phase warp r owns row r.
// dynamic smem: qs[rows][D] + ks[D][kSelTile + 1] + pz[8][rows][32] + z[rows][nr]
//               + e[rows][nr]
template <int D>
__global__ void __launch_bounds__(256) nabla_select_kernel(
    const float* __restrict__ qbar, const float* __restrict__ kbar, int heads, int qb_count,
    int kb_count, int kb_begin, int kb_end, float p, float scale, int force_outside,
    const uint8_t* __restrict__ base_mask, const uint8_t* __restrict__ key_allowed,
    uint8_t* __restrict__ mask, int* __restrict__ near_count, int rows) {
  extern __shared__ float smem[];
  const int nr = kb_end - kb_begin;
  constexpr int kKs = kSelTile + 1;        // transposed key tile row (conflict-free)
  constexpr int DW = D / kSelRows;         // head_dim columns per warp
  float* qs = smem;
  float* ks = qs + rows * D;
  float* pz = ks + D * kKs;
  float* zs = pz + kSelRows * rows * 32;
  float* es = zs + rows * nr;
  const int b = blockIdx.z, h = blockIdx.y;
  const int q0 = blockIdx.x * rows;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* qsrc = qbar + (static_cast<long long>(b) * heads + h) * qb_count * D;
  const float* ksrc = kbar + (static_cast<long long>(b) * heads + h) * kb_count * D;

  for (int i = tid; i < rows * D; i += blockDim.x) {
    const int r = i / D;
    qs[i] = (q0 + r < qb_count) ? qsrc[static_cast<long long>(q0 + r) * D + (i - r * D)] : 0.f;
  }
  // logits z[r][c] = qbar[r] . kbar[kb_begin + c] * scale
  const int j0 = warp * DW;
  for (int t0 = 0; t0 < nr; t0 += kSelTile) {
    __syncthreads();   // the previous tile's keys and partials are consumed
    for (int i = tid; i < kSelTile * D; i += blockDim.x) {
      const int c = i / D, j = i - c * D;
      ks[j * kKs + c] =
          (t0 + c < nr) ? ksrc[static_cast<long long>(kb_begin + t0 + c) * D + j] : 0.f;
    }
    __syncthreads();
    float acc[kSelRows];
#pragma unroll
    for (int r = 0; r < kSelRows; ++r) acc[r] = 0.f;
#pragma unroll
    for (int j = j0; j < j0 + DW; j += 4) {
      const float k0 = ks[j * kKs + lane], k1 = ks[(j + 1) * kKs + lane];
      const float k2 = ks[(j + 2) * kKs + lane], k3 = ks[(j + 3) * kKs + lane];
#pragma unroll
      for (int r = 0; r < kSelRows; ++r) {
        if (r < rows) {
          const float4 qv = *reinterpret_cast<const float4*>(qs + r * D + j);
          acc[r] = fmaf(qv.x, k0, acc[r]);
          acc[r] = fmaf(qv.y, k1, acc[r]);
          acc[r] = fmaf(qv.z, k2, acc[r]);
          acc[r] = fmaf(qv.w, k3, acc[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kSelRows; ++r)
      if (r < rows) pz[(warp * rows + r) * 32 + lane] = acc[r];
    __syncthreads();
    for (int i = tid; i < rows * 32; i += blockDim.x) {
      const int r = i >> 5, c = i & 31;
      if (t0 + c < nr) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kSelRows; ++w) sum += pz[(w * rows + r) * 32 + c];
        zs[r * nr + t0 + c] = sum * scale;
      }
    }
  }
  __syncthreads();

  if (warp >= rows) return;
  const int qb = q0 + warp;
  if (qb >= qb_count) return;
  uint8_t* mrow = mask + ((static_cast<long long>(b) * heads + h) * qb_count + qb) * kb_count;
  // optional head-shared mask OR-ed into the result (e.g. a Sliding-Tile window)
  const uint8_t* brow = base_mask ? base_mask + static_cast<long long>(qb) * kb_count : nullptr;
  const uint8_t fo = force_outside ? 1 : 0;
  for (int c = lane; c < kb_begin; c += 32) mrow[c] = fo | (brow ? (brow[c] != 0) : 0);
  for (int c = kb_end + lane; c < kb_count; c += 32) mrow[c] = fo | (brow ? (brow[c] != 0) : 0);
  if (nr <= 0) return;

  float* z = zs + warp * nr;
  float* e = es + warp * nr;
  // key blocks that may not be chosen (evicted from a paged cache) leave the softmax
  const uint8_t* arow = key_allowed ? key_allowed + static_cast<long long>(b) * kb_count + kb_begin
                                    : nullptr;
  if (arow) {
    for (int c = lane; c < nr; c += 32)
      if (!arow[c]) z[c] = -INFINITY;
    __syncwarp();
  }
  float m = -INFINITY;
  for (int c = lane; c < nr; c += 32) m = fmaxf(m, z[c]);
  m = warp_max(m);
  if (m == -INFINITY) {  // no candidate: only the base mask
    for (int c = lane; c < nr; c += 32) mrow[kb_begin + c] = (brow && brow[kb_begin + c] != 0) ? 1 : 0;
    return;
  }
  float tot = 0.f;
  for (int c = lane; c < nr; c += 32) {
    const float v = __expf(z[c] - m);
    e[c] = v;
    tot += v;
  }
  tot = warp_sum(tot);
  __syncwarp();

  if (p >= 1.0f) {
    for (int c = lane; c < nr; c += 32)
      mrow[kb_begin + c] = (!arow || arow[c] || (brow && brow[kb_begin + c] != 0)) ? 1 : 0;
    return;
  }
  const float target = p * tot;
  // largest v with F(v) = sum_{key_c >= v} e_c >= target
  const uint32_t v = nr <= 32 * 16 ? radix_cut_regs<16>(z, e, nr, lane, target)
                                   : radix_cut(z, e, nr, lane, target);
  // mass strictly above the cut, the tied value, and the largest value below it
  float f_gt = 0.f, e_eq = 0.f, e_below = 0.f;
  int n_eq = 0;
  for (int c = lane; c < nr; c += 32) {
    const uint32_t key = order_key(z[c]);
    if (key > v) f_gt += e[c];
    else if (key == v) { e_eq = e[c]; ++n_eq; }
    else e_below = fmaxf(e_below, e[c]);
  }
  f_gt = warp_sum(f_gt);
  e_eq = warp_max(e_eq);
  e_below = warp_max(e_below);
  n_eq = warp_isum(n_eq);
  int t = 1;
  float cum = f_gt + e_eq;
  while (cum < target && t < n_eq) {
    ++t;
    cum += e_eq;
  }
  // kept: key > v, plus the first t tied entries in index order
  int ties_seen = 0;
  for (int c0 = 0; c0 < nr; c0 += 32) {
    const int c = c0 + lane;
    uint32_t key = 0;
    if (c < nr) key = order_key(z[c]);
    const bool tie = c < nr && key == v;
    const uint32_t bal = __ballot_sync(0xffffffffu, tie);
    const int rank = ties_seen + __popc(bal & ((1u << lane) - 1u));
    ties_seen += __popc(bal);
    if (c < nr)
      mrow[kb_begin + c] = ((key > v || (tie && rank < t)) || (brow && brow[kb_begin + c] != 0)) ? 1 : 0;
  }
  if (lane == 0 && near_count) {
    const float c_last = cum / tot, c_prev = (cum - e_eq) / tot;
    bool near = fabsf(c_last - p) < 1e-5f || fabsf(c_prev - p) < 1e-5f;
    if (t == n_eq && e_below > 0.f && e_below >= e_eq * (1.0f - 1e-5f)) near = true;
    if (near) atomicAdd(near_count, 1);
  }
}

size_t nabla_ws_bytes(int batch, int heads, int nq, int nk, int head_dim, int block) {
  const size_t qb = ceil_div(nq, block), kb = ceil_div(nk, block);
  return kStatusBytes + sizeof(float) * static_cast<size_t>(batch) * heads * head_dim * (qb + kb);
}

}  // namespace
}  // namespace bsa

extern "C" size_t bsa_nabla_workspace_size(int batch, int heads, int nq, int nk, int head_dim,
                                           int block) {
  if (batch < 1 || heads < 1 || nq < 1 || nk < 1 || head_dim < 1 || block < 1) return 0;
  return bsa::nabla_ws_bytes(batch, heads, nq, nk, head_dim, block);
}

namespace bsa {
namespace {

// Shared memory of the selection kernel for `rows` query rows per CTA.
size_t select_smem(int rows, int head_dim, int nr) {
  return sizeof(float) * (static_cast<size_t>(rows) * head_dim +
                          static_cast<size_t>(head_dim) * (kSelTile + 1) +
                          static_cast<size_t>(kSelRows) * rows * 32 +
                          2 * static_cast<size_t>(rows) * nr);
}

constexpr size_t kSelSmemLimit = 200 * 1024;

int launch_select(const float* qbar, const float* kbar, int batch, int heads, int qb, int kb,
                  int head_dim, float p, float scale, int kb_begin, int kb_end, int force_outside,
                  const uint8_t* base_mask, const uint8_t* key_allowed, uint8_t* mask,
                  int* near_count, cudaStream_t st) {
  const int nr = kb_end - kb_begin;
  // as many rows per CTA as the rows' logits allow (8 up to ~2,900 candidate key
  // blocks at head_dim 128, 1 up to ~23,000)
  int rows = kSelRows;
  while (rows > 1 && select_smem(rows, head_dim, nr) > kSelSmemLimit) rows >>= 1;
  const size_t smem = select_smem(rows, head_dim, nr);
  if (smem > kSelSmemLimit) return BSA_ERR_UNSUPPORTED;
  if (scale <= 0.0f) scale = 1.0f / sqrtf(static_cast<float>(head_dim));
  if (near_count) {
    cudaError_t e = cudaMemsetAsync(near_count, 0, sizeof(int), st);
    if (e != cudaSuccess) return record_cuda_error(e);
  }
  dim3 sgrid(ceil_div(qb, rows), heads, batch);
  // the shared-memory cap is raised to the selection's limit once per device (not
  // per launch, so that a launch can be captured into a CUDA graph)
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nabla_select_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSelSmemLimit));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(nabla_select_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kSelSmemLimit));
    if (e != cudaSuccess) return record_cuda_error(e);
    if (dev >= 0 && dev < 64) attr_done[dev] = true;
  }
  if (head_dim == 128) {
    nabla_select_kernel<128><<<sgrid, 256, smem, st>>>(qbar, kbar, heads, qb, kb, kb_begin, kb_end,
                                                       p, scale, force_outside, base_mask, key_allowed, mask,
                                                       near_count, rows);
  } else {
    nabla_select_kernel<64><<<sgrid, 256, smem, st>>>(qbar, kbar, heads, qb, kb, kb_begin, kb_end,
                                                      p, scale, force_outside, base_mask, key_allowed, mask,
                                                      near_count, rows);
  }
  return check_launch();
}

}  // namespace
}  // namespace bsa

extern "C" int bsa_nabla_select(const float* qbar, const float* kbar, int batch, int heads,
                                int QB, int KB, int head_dim, float p, float scale, int kb_begin,
                                int kb_end, int force_outside, const uint8_t* base_mask,
                                const uint8_t* key_allowed, uint8_t* mask, int* near_count,
                                void* stream) {
  BSA_NVTX_RANGE("bsa_nabla_select");
  using namespace bsa;
  if (!qbar || !kbar || !mask) return BSA_ERR_INVALID_ARG;
  if (batch < 1 || heads < 1 || QB < 1 || KB < 1 || !(p > 0.0f)) return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (kb_begin < 0 || kb_end > KB || kb_begin > kb_end) return BSA_ERR_INVALID_ARG;
  return launch_select(qbar, kbar, batch, heads, QB, KB, head_dim, p, scale, kb_begin, kb_end,
                       force_outside, base_mask, key_allowed, mask, near_count,
                       static_cast<cudaStream_t>(stream));
}

extern "C" int bsa_nabla_mask(const void* q, const void* k, int batch, int heads, int nq, int nk,
                              int head_dim, int row_stride, int block, float p, float scale,
                              int kb_begin, int kb_end, int force_outside, uint8_t* mask,
                              int* near_count, void* ws, size_t ws_bytes, void* stream) {
  BSA_NVTX_RANGE("bsa_nabla_mask");
  using namespace bsa;
  if (!q || !k || !mask || !ws) return BSA_ERR_INVALID_ARG;
  if (batch < 1 || heads < 1 || nq < 1 || nk < 1 || block < 16 || block > 1024 ||
      (block % 16) != 0 || !(p > 0.0f))
    return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(ws)) return BSA_ERR_INVALID_ARG;
  const long long dense = static_cast<long long>(heads) * head_dim;
  const long long rs = row_stride == 0 ? dense : row_stride;
  if (rs < dense || (rs % 8) != 0) return BSA_ERR_INVALID_ARG;
  const int qb = ceil_div(nq, block), kb = ceil_div(nk, block);
  if (kb_begin < 0 || kb_end > kb || kb_begin > kb_end) return BSA_ERR_INVALID_ARG;
  if (ws_bytes < nabla_ws_bytes(batch, heads, nq, nk, head_dim, block)) return BSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* qbar = reinterpret_cast<float*>(static_cast<char*>(ws) + kStatusBytes);
  float* kbar = qbar + static_cast<size_t>(batch) * heads * qb * head_dim;
  const int C = heads * head_dim;
  dim3 pgrid(qb > kb ? qb : kb, ceil_div(C, kPoolCols), batch * 2);
  nabla_pool_kernel<<<pgrid, kPoolThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), heads,
      head_dim, rs, nq, nk, block, qb, kb, qbar, kbar);
  int rc = check_launch();
  if (rc != BSA_OK) return rc;
  return launch_select(qbar, kbar, batch, heads, qb, kb, head_dim, p, scale, kb_begin, kb_end,
                       force_outside, nullptr, nullptr, mask, near_count, st);
}
