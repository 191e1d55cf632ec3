// lserve_quantize_pages_kv8 / _kv4 kernel: an 8-bit or 4-bit copy of the
// paged K / V cache with one float32 scale per (pool page, KV head, channel)
// (the quantized KV cache the LServe abstract page combines with the unified
// sparsity; the pages give no scheme, so this library uses symmetric
// per-page, per-channel codes: -127..127, or -7..7 packed two per byte, the
// even channel in the low nibble).
//
// One CTA of 128 threads per (page of a sequence, KV head, tensor K or V).
// D/8 threads cover a row with 16-byte loads; the row groups of the CTA walk
// the page's valid rows twice: first for the channel's largest magnitude
// (exact in float32), reduced across the row groups in shared memory, then to
// turn every value into its code.  The second read hits L1 (the page is at
// most N_P * D * 2 bytes, read by the same threads a moment earlier).
// Decisions in float32, IEEE-rounded, in this order (Q = 127 or 7):
//   amax_c  = max_t |x[t][c]|
//   inv_c   = Q / amax_c              (0 when amax_c == 0)
//   code    = rint(x * inv_c), clamped to [-Q, Q]   (half to even)
//   scale_c = amax_c / Q
// Rows past the page's valid tokens get code 0.  HBM-bound: the bf16 page is
// read once from DRAM, the codes (half its size) and 4*D bytes of scales are
// written.
#include "common.cuh"
#include "kernels.h"

namespace lserve {

namespace {
constexpr int kQuantThreads = 128;
}

template <int D, int BITS>
__global__ void __launch_bounds__(kQuantThreads) quantize_kv_kernel(QuantParams p) {
  constexpr float Q = BITS == 8 ? 127.f : 7.f;
  constexpr int QI = BITS == 8 ? 127 : 7;
  constexpr int RB = D * BITS / 8;           // code bytes per row
  constexpr int TPR = D / 8;                 // threads per row (8 channels each)
  constexpr int RG = kQuantThreads / TPR;    // row groups
  __shared__ float red[RG][D];
  __shared__ float inv_s[D];
  const int tid = threadIdx.x;
  const int rg = tid / TPR, cq = tid % TPR;
  const int slot = blockIdx.x;               // b * max_pages + m
  const int h = blockIdx.y;
  const bool is_v = blockIdx.z != 0;
  const int b = slot / p.max_pages, m = slot - b * p.max_pages;
  const int NP = p.physical_page;
  const int n = p.ctx_lens[b];
  if ((long long)m * NP >= n) return;        // page past the sequence: nothing to do
  const int pid = p.block_table[(size_t)b * p.max_pages + m];
  if (pid < 0 || pid >= p.num_pool_pages) {
    if (tid == 0) raise_status(p.status, LSERVE_ERR_BOUNDS);
    return;
  }
  const int valid = min(NP, n - m * NP);
  const size_t base = ((size_t)pid * p.num_kv_heads + h) * NP;  // first row of (page, head)
  const __nv_bfloat16* src = (is_v ? p.v_pool : p.k_pool) + base * D + cq * 8;
  int8_t* dst = (is_v ? p.v_pool8 : p.k_pool8) + base * RB + cq * BITS;
  float* scale_out = (is_v ? p.v_scale : p.k_scale) + ((size_t)pid * p.num_kv_heads + h) * D;

  // pass 1: largest magnitude of this thread's 8 channels over its rows
  float am[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) am[i] = 0.f;
  for (int r = rg; r < valid; r += RG) {
    const uint4 w = *reinterpret_cast<const uint4*>(src + (size_t)r * D);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      am[2 * i] = fmaxf(am[2 * i], fabsf(bf16_lo(ws[i])));
      am[2 * i + 1] = fmaxf(am[2 * i + 1], fabsf(bf16_hi(ws[i])));
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[rg][cq * 8 + i] = am[i];
  __syncthreads();
  for (int c = tid; c < D; c += kQuantThreads) {
    float a = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) a = fmaxf(a, red[g][c]);
    inv_s[c] = a > 0.f ? __fdiv_rn(Q, a) : 0.f;
    scale_out[c] = __fdiv_rn(a, Q);
  }
  __syncthreads();

  // pass 2: codes (valid rows), zeros (the rest of the page)
  float inv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) inv[i] = inv_s[cq * 8 + i];
  for (int r = rg; r < NP; r += RG) {
    uint32_t packed[2] = {0u, 0u};  // 8 codes: 8 bytes, or 8 nibbles in packed[0]
    if (r < valid) {
      const uint4 w = *reinterpret_cast<const uint4*>(src + (size_t)r * D);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float x = (i & 1) ? bf16_hi(ws[i / 2]) : bf16_lo(ws[i / 2]);
        int c = __float2int_rn(__fmul_rn(x, inv[i]));
        c = max(-QI, min(QI, c));
        if constexpr (BITS == 8) packed[i / 4] |= ((uint32_t)c & 0xFFu) << (8 * (i % 4));
        else packed[0] |= ((uint32_t)c & 0xFu) << (4 * i);
      }
    }
    if constexpr (BITS == 8)
      *reinterpret_cast<uint2*>(dst + (size_t)r * RB) = make_uint2(packed[0], packed[1]);
    else
      *reinterpret_cast<uint32_t*>(dst + (size_t)r * RB) = packed[0];
  }
}

cudaError_t launch_quantize_kv(const QuantParams& p, int D, int bits, cudaStream_t stream) {
  const long long slots = (long long)p.batch * p.max_pages;
  if (slots < 1 || slots > 0x7fffffffll || p.num_kv_heads > 65535) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)slots, (unsigned)p.num_kv_heads, 2);
  if (D == 128 && bits == 8) {
    quantize_kv_kernel<128, 8><<<grid, kQuantThreads, 0, stream>>>(p);
  } else if (D == 64 && bits == 8) {
    quantize_kv_kernel<64, 8><<<grid, kQuantThreads, 0, stream>>>(p);
  } else if (D == 128 && bits == 4) {
    quantize_kv_kernel<128, 4><<<grid, kQuantThreads, 0, stream>>>(p);
  } else if (D == 64 && bits == 4) {
    quantize_kv_kernel<64, 4><<<grid, kQuantThreads, 0, stream>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace lserve
