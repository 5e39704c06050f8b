// fa_append_kernel.cu -- writes new K/V tokens into the paged caches
// ("Flash-Attention v2.0 到 v2.7 更新", v2.5: the cache lives in pages reached
// through block_table; "解密FlashAttention：如何让大语言模型推理速度翻倍",
// section 智能緩存機制: the key-value cache keeps the context already
// processed, so each decoding step adds its keys and values to it). Token t
// of sequence b lives in row t % page_size of page
// block_table[b][t / page_size]; the n_new new tokens of sequence b take the
// positions cache_seqlens[b] .. cache_seqlens[b] + n_new - 1.
#include "fa_internal.h"

namespace fa {
namespace {

// One thread per 16-byte chunk of one (sequence, new token, head) row; K and
// V rows are copied by the same thread. Positions past the table or pages
// out of range are skipped (nothing is written for them).
__global__ void append_kernel(const AppendParams p) {
  const int chunks = p.d / 8;  // 16-byte chunks of a 16-bit row
  const long long total = static_cast<long long>(p.B) * p.n_new * p.H_kv * chunks;
  const long long cap = static_cast<long long>(p.max_blocks) * p.page_size;
  for (long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx % chunks);
    long long r = idx / chunks;
    const int h = static_cast<int>(r % p.H_kv);
    r /= p.H_kv;
    const int i = static_cast<int>(r % p.n_new);
    const int b = static_cast<int>(r / p.n_new);
    const int L = p.cache_seqlens[b];
    const long long t = static_cast<long long>(L) + i;
    if (L < 0 || t >= cap) continue;
    const int pg = p.block_table[static_cast<size_t>(b) * p.max_blocks + static_cast<size_t>(t / p.page_size)];
    if (pg < 0 || pg >= p.num_pages) continue;
    const size_t src = ((static_cast<size_t>(b) * p.n_new + i) * p.H_kv + h) * p.d + static_cast<size_t>(c) * 8;
    const size_t dst = ((static_cast<size_t>(pg) * p.page_size + static_cast<size_t>(t % p.page_size)) * p.H_kv + h) *
                           p.d +
                       static_cast<size_t>(c) * 8;
    // 16-bit elements: 8 per 16-byte chunk
    const uint4* ks = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.k_new) + src);
    const uint4* vs = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.v_new) + src);
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.k_cache) + dst) = *ks;
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.v_cache) + dst) = *vs;
  }
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
  const long long total = static_cast<long long>(p.B) * p.n_new * p.H_kv * (p.d / 8);
  const long long want = (total + 255) / 256;
  const unsigned blocks = static_cast<unsigned>(want < 148 * 16 ? want : 148 * 16);
  append_kernel<<<blocks, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace fa
