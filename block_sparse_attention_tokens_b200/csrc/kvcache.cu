// Paged KV cache with persistent anchors for autoregressive chunk decoding.
//
// Source: the Sparse Forcing summary (gist.science/ja/paper/2604.21221), part 2
// (the anchors -- who and where -- are kept as persistent memory, the recent
// frames are looked at closely with only the needed parts, and the past is not
// stored whole: only its important points are kept, cutting the memory) and
// part 4 (memory use down by 42 %).
//
// K and V live in a pool of 128-token pages (one attention k-tile each); a page
// table per batch maps logical page -> physical page, -1 once evicted.  After a
// chunk, every page's importance is the pooled attention probability the chunk's
// queries put on it (the distribution NABLA selects from, summed over heads and
// query blocks); the cache keeps the anchor pages, the recent pages and a fixed
// budget of the most important pages in between, and frees the rest.
#include "bsa_common.cuh"
#include "nvtx_range.cuh"

#include <cuda_bf16.h>

namespace bsa {
namespace {

constexpr int kPage = 128;           // tokens per page
constexpr int kPoolThreads = 128;    // 8 columns per thread
constexpr int kMaxSortPages = 8192;  // middle pages ranked by one CTA

// One warp per token row: row i of batch b goes to logical token first + i.
__global__ void kv_write_kernel(const uint4* __restrict__ src, int batch, int n_new, int row_vec,
                                int first, const int* __restrict__ page_table, int pages_per_batch,
                                int n_pool_pages, uint4* __restrict__ pool, int* status) {
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<long long>(batch) * n_new) return;
  const int b = static_cast<int>(wid / n_new), i = static_cast<int>(wid - static_cast<long long>(b) * n_new);
  const int t = first + i;
  const int lp = t / kPage;
  const int page = lp < pages_per_batch ? page_table[static_cast<long long>(b) * pages_per_batch + lp] : -1;
  if (page < 0 || page >= n_pool_pages) {
    if (lane == 0 && status) set_status(status, BSA_ERR_INVALID_ARG);
    return;
  }
  const uint4* s = src + wid * row_vec;
  uint4* d = pool + (static_cast<long long>(page) * kPage + (t - lp * kPage)) * row_vec;
  for (int c = lane; c < row_vec; c += 32) d[c] = __ldg(s + c);
}

// grid: x = block (relative to first_block), y = column chunk of 8 * kPoolThreads,
// z = batch.  Mean of the block's tokens below n_tokens, per column (head x dim).
__global__ void __launch_bounds__(kPoolThreads) block_pool_kernel(
    const __nv_bfloat16* __restrict__ x, const int* __restrict__ page_table, int pages_per_batch,
    int n_tokens, int heads, int head_dim, int block, int first_block, int out_blocks,
    float* __restrict__ out) {
  const int blk = first_block + blockIdx.x;
  const int b = blockIdx.z;
  const int C = heads * head_dim;
  const int col = (blockIdx.y * kPoolThreads + threadIdx.x) * 8;
  if (col >= C) return;
  const int r0 = blk * block, r1 = min(r0 + block, n_tokens);
  if (r1 <= r0) return;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int r = r0; r < r1; ++r) {
    long long row;
    if (page_table) {
      const int page = page_table[static_cast<long long>(b) * pages_per_batch + r / kPage];
      if (page < 0) continue;  // an evicted page reads as zero
      row = static_cast<long long>(page) * kPage + (r % kPage);
    } else {
      row = static_cast<long long>(b) * n_tokens + r;
    }
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + row * C + col));
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(p2[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
  const float inv = 1.0f / static_cast<float>(r1 - r0);
  const int h = col / head_dim, j = col - h * head_dim;
  float4* o = reinterpret_cast<float4*>(
      out + ((static_cast<long long>(b) * heads + h) * out_blocks + blk) * head_dim + j);
  o[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  o[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
}

// key_allowed[b][kb] = 1 iff the page holding key block kb is resident.
__global__ void resident_blocks_kernel(const int* __restrict__ page_table, int batch,
                                       int pages_per_batch, int block, int KB,
                                       uint8_t* __restrict__ allowed) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<long long>(batch) * KB) return;
  const int b = static_cast<int>(i / KB), kb = static_cast<int>(i - static_cast<long long>(b) * KB);
  const int lp = (kb * block) / kPage;
  allowed[i] = (lp < pages_per_batch &&
                page_table[static_cast<long long>(b) * pages_per_batch + lp] >= 0) ? 1 : 0;
}

// grid: x = query block, y = head, z = batch; 128 threads.  Softmax of the pooled
// logits over the candidate key blocks, each block's probability added to its page.
// dynamic smem: z[nr] floats + page sums [n_range_pages] floats + qbar row [D].
template <int D>
__global__ void __launch_bounds__(128) page_scores_kernel(
    const float* __restrict__ qbar, const float* __restrict__ kbar, int heads, int QB, int KB,
    float scale, int kb_begin, int kb_end, const uint8_t* __restrict__ key_allowed, int block,
    int n_pages, float* __restrict__ scores) {
  extern __shared__ float sm[];
  const int nr = kb_end - kb_begin;
  const int p_first = (kb_begin * block) / kPage;
  const int p_count = ((kb_end - 1) * block) / kPage - p_first + 1;
  float* z = sm;
  float* ps = z + nr;
  float* qs = ps + p_count;
  __shared__ float red[4];
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* qrow = qbar + ((static_cast<long long>(b) * heads + h) * QB + qb) * D;
  const float* kb0 = kbar + (static_cast<long long>(b) * heads + h) * KB * D;
  for (int i = tid; i < D; i += 128) qs[i] = qrow[i];
  for (int i = tid; i < p_count; i += 128) ps[i] = 0.f;
  __syncthreads();
  for (int c = warp; c < nr; c += 4) {
    const int kb = kb_begin + c;
    const bool ok = !key_allowed || key_allowed[static_cast<long long>(b) * KB + kb];
    float acc = 0.f;
    if (ok) {
      const float* kr = kb0 + static_cast<long long>(kb) * D;
#pragma unroll
      for (int j = lane; j < D; j += 32) acc = fmaf(qs[j], kr[j], acc);
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) z[c] = ok ? acc * scale : -INFINITY;
  }
  __syncthreads();
  float m = -INFINITY;
  for (int c = tid; c < nr; c += 128) m = fmaxf(m, z[c]);
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  if (m == -INFINITY) return;  // no candidate block
  float tot = 0.f;
  for (int c = tid; c < nr; c += 128) {
    const float e = __expf(z[c] - m);
    z[c] = e;
    tot += e;
  }
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  if (lane == 0) red[warp] = tot;
  __syncthreads();
  tot = (red[0] + red[1]) + (red[2] + red[3]);
  const float inv = 1.0f / tot;
  for (int c = tid; c < nr; c += 128)
    if (z[c] > 0.f) atomicAdd(&ps[((kb_begin + c) * block) / kPage - p_first], z[c] * inv);
  __syncthreads();
  for (int i = tid; i < p_count; i += 128)
    if (ps[i] != 0.f && p_first + i < n_pages)
      atomicAdd(&scores[static_cast<long long>(b) * n_pages + p_first + i], ps[i]);
}

// One CTA per batch: rank the resident middle pages by (score desc, page asc) with
// a bitonic sort in shared memory, keep the first `budget`, evict the rest (page
// table entry -1, physical page appended to the freed list).
__global__ void __launch_bounds__(1024) keep_pages_kernel(
    const float* __restrict__ scores, int n_pages, int anchor_pages, int recent_begin, int budget,
    int* __restrict__ page_table, int pages_per_batch, int* __restrict__ freed,
    int* __restrict__ freed_count) {
  extern __shared__ unsigned long long keys[];
  const int b = blockIdx.x;
  const int n_mid = recent_begin - anchor_pages;
  int n2 = 1;
  while (n2 < n_mid) n2 <<= 1;
  int* pt = page_table + static_cast<long long>(b) * pages_per_batch;
  const float* sc = scores + static_cast<long long>(b) * n_pages;
  for (int i = threadIdx.x; i < n2; i += blockDim.x) {
    unsigned long long key = 0ull;
    if (i < n_mid) {
      const int pg = anchor_pages + i;
      if (pt[pg] >= 0) {
        // scores are >= 0, so their bit patterns order like the values; + 1 keeps a
        // resident page with score 0 above the empty slots
        const unsigned long long s = static_cast<unsigned long long>(__float_as_uint(fmaxf(sc[pg], 0.f))) + 1ull;
        key = (s << 32) | static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(pg));
      }
    }
    keys[i] = key;
  }
  __syncthreads();
  // bitonic sort, descending
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        const int l = i ^ j;
        if (l > i) {
          const bool desc = (i & k) == 0;
          const unsigned long long a = keys[i], c = keys[l];
          if (desc ? (a < c) : (a > c)) {
            keys[i] = c;
            keys[l] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = budget + threadIdx.x; i < n_mid; i += blockDim.x) {
    const unsigned long long key = keys[i];
    if (key == 0ull) continue;  // not resident
    const int pg = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(key & 0xFFFFFFFFull));
    const int phys = pt[pg];
    pt[pg] = -1;
    freed[atomicAdd(freed_count, 1)] = phys;
  }
}

}  // namespace
}  // namespace bsa

extern "C" int bsa_kv_write(const void* src, int batch, int n_new, int heads, int head_dim,
                            int first_token, const int* page_table, int pages_per_batch,
                            void* pool, int n_pool_pages, int* device_status, void* stream) {
  BSA_NVTX_RANGE("bsa_kv_write");
  using namespace bsa;
  if (!src || !page_table || !pool || !aligned16(src) || !aligned16(pool)) return BSA_ERR_INVALID_ARG;
  if (batch < 1 || n_new < 1 || heads < 1 || first_token < 0 || pages_per_batch < 1 ||
      n_pool_pages < 1)
    return BSA_ERR_INVALID_ARG;
  if ((heads * head_dim) % 8 != 0 || head_dim < 8) return BSA_ERR_UNSUPPORTED;
  if (ceil_div(first_token + n_new, kPage) > pages_per_batch) return BSA_ERR_INVALID_ARG;
  const long long warps = static_cast<long long>(batch) * n_new;
  const long long blocks = (warps * 32 + 255) / 256;
  if (blocks > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
  kv_write_kernel<<<static_cast<int>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), batch, n_new, heads * head_dim / 8, first_token, page_table,
      pages_per_batch, n_pool_pages, static_cast<uint4*>(pool), device_status);
  return check_launch();
}

extern "C" int bsa_block_pool(const void* x, const int* page_table, int pages_per_batch, int batch,
                              int n_tokens, int heads, int head_dim, int block, int first_block,
                              int n_blocks, float* out, int out_blocks, void* stream) {
  BSA_NVTX_RANGE("bsa_block_pool");
  using namespace bsa;
  if (!x || !out || !aligned16(x)) return BSA_ERR_INVALID_ARG;
  if (batch < 1 || n_tokens < 1 || heads < 1 || block < 1 || first_block < 0 || n_blocks < 1 ||
      first_block + n_blocks > out_blocks || (first_block + n_blocks - 1) * static_cast<long long>(block) >= n_tokens)
    return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (page_table && ceil_div(n_tokens, kPage) > pages_per_batch) return BSA_ERR_INVALID_ARG;
  const int C = heads * head_dim;
  dim3 grid(n_blocks, ceil_div(C, 8 * kPoolThreads), batch);
  if (batch > 65535) return BSA_ERR_UNSUPPORTED;
  block_pool_kernel<<<grid, kPoolThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), page_table, pages_per_batch, n_tokens, heads, head_dim,
      block, first_block, out_blocks, out);
  return check_launch();
}

extern "C" int bsa_kv_resident_blocks(const int* page_table, int batch, int pages_per_batch,
                                      int block, int KB, uint8_t* allowed, void* stream) {
  BSA_NVTX_RANGE("bsa_kv_resident_blocks");
  using namespace bsa;
  if (!page_table || !allowed || batch < 1 || pages_per_batch < 1 || block < 1 || KB < 1)
    return BSA_ERR_INVALID_ARG;
  if (kPage % block != 0) return BSA_ERR_UNSUPPORTED;
  const long long n = static_cast<long long>(batch) * KB;
  resident_blocks_kernel<<<static_cast<int>((n + 255) / 256), 256, 0,
                           static_cast<cudaStream_t>(stream)>>>(page_table, batch, pages_per_batch,
                                                                block, KB, allowed);
  return check_launch();
}

extern "C" int bsa_kv_page_scores(const float* qbar, const float* kbar, int batch, int heads,
                                  int QB, int KB, int head_dim, float scale, int kb_begin,
                                  int kb_end, const uint8_t* key_allowed, int block, int n_pages,
                                  float* scores, void* stream) {
  BSA_NVTX_RANGE("bsa_kv_page_scores");
  using namespace bsa;
  if (!qbar || !kbar || !scores || batch < 1 || heads < 1 || QB < 1 || KB < 1 || n_pages < 1)
    return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (kb_begin < 0 || kb_end > KB || kb_begin > kb_end || block < 1 || kPage % block != 0)
    return BSA_ERR_INVALID_ARG;
  if (heads > 65535 || batch > 65535) return BSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(scores, 0, sizeof(float) * static_cast<size_t>(batch) * n_pages, st);
  if (e != cudaSuccess) return record_cuda_error(e);
  const int nr = kb_end - kb_begin;
  if (nr == 0) return BSA_OK;
  const int p_count = ((kb_end - 1) * block) / kPage - (kb_begin * block) / kPage + 1;
  const size_t smem = sizeof(float) * (static_cast<size_t>(nr) + p_count + head_dim);
  if (smem > 200 * 1024) return BSA_ERR_UNSUPPORTED;
  dim3 grid(QB, heads, batch);
  if (head_dim == 128) {
    if (smem > 48 * 1024 &&
        (e = cudaFuncSetAttribute(page_scores_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(smem))) != cudaSuccess)
      return record_cuda_error(e);
    page_scores_kernel<128><<<grid, 128, smem, st>>>(qbar, kbar, heads, QB, KB, scale, kb_begin,
                                                     kb_end, key_allowed, block, n_pages, scores);
  } else {
    if (smem > 48 * 1024 &&
        (e = cudaFuncSetAttribute(page_scores_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(smem))) != cudaSuccess)
      return record_cuda_error(e);
    page_scores_kernel<64><<<grid, 128, smem, st>>>(qbar, kbar, heads, QB, KB, scale, kb_begin,
                                                    kb_end, key_allowed, block, n_pages, scores);
  }
  return check_launch();
}

extern "C" int bsa_kv_keep_pages(const float* scores, int batch, int n_pages, int anchor_pages,
                                 int recent_begin, int budget, int* page_table,
                                 int pages_per_batch, int* freed, int* freed_count, void* stream) {
  BSA_NVTX_RANGE("bsa_kv_keep_pages");
  using namespace bsa;
  if (!scores || !page_table || !freed || !freed_count || batch < 1 || n_pages < 1 ||
      budget < 0 || anchor_pages < 0 || recent_begin > n_pages || anchor_pages > recent_begin ||
      pages_per_batch < n_pages)
    return BSA_ERR_INVALID_ARG;
  const int n_mid = recent_begin - anchor_pages;
  if (n_mid > kMaxSortPages) return BSA_ERR_UNSUPPORTED;
  if (n_mid == 0) return BSA_OK;
  int n2 = 1;
  while (n2 < n_mid) n2 <<= 1;
  const size_t smem = sizeof(unsigned long long) * n2;
  cudaError_t e = cudaSuccess;
  if (smem > 48 * 1024 &&
      (e = cudaFuncSetAttribute(keep_pages_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smem))) != cudaSuccess)
    return record_cuda_error(e);
  keep_pages_kernel<<<batch, 1024, smem, static_cast<cudaStream_t>(stream)>>>(
      scores, n_pages, anchor_pages, recent_begin, budget, page_table, pages_per_batch, freed,
      freed_count);
  return check_launch();
}
