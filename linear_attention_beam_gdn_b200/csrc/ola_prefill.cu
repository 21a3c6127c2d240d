// Prompt prefill: the shared post-prefill state of every (request, head).
//
// "Scientific Impact Assessment: OneLA", §1 Core Contribution: all beams of a request start
// from one recurrent state derived from the shared prompt. The state is produced by applying
// the gated delta rule token by token from S = 0:
//     u = S k,  w = beta (v - alpha u),  S <- alpha S + w k^T      (alpha = exp(g))
// which is alpha S (I - beta k k^T) + beta v k^T rewritten with S (k k^T) = (S k) k^T.
//
// Row i of S only ever meets v_i and the shared key: rows are independent. Each thread keeps
// a SEG-wide slice of one row in registers for the whole prompt; TPR = d_k / SEG threads
// share a row and combine u with lane shuffles. Prompt tokens are staged in shared memory 32
// at a time. The kernel is compute-light and runs once per request batch (not per decode
// step).
#include "ola_device.cuh"

namespace ola {

constexpr int kPrefillThreads = 256;
constexpr int kTokChunk = 32;

template <typename TIn>
__global__ void __launch_bounds__(kPrefillThreads)
prefill_kernel(int R, int H, int d_k, int d_v, int P, const void* __restrict__ kp,
               const void* __restrict__ vp, const float* __restrict__ gp,
               const float* __restrict__ bp, float* __restrict__ S_out) {
  extern __shared__ float smem[];
  const int SEG = d_k < 32 ? d_k : 32;
  const int TPR = d_k / SEG;                       // threads per row (power of two <= 8)
  const int rows_cta = kPrefillThreads / TPR;
  const int kstride = d_k + TPR;                   // pad each SEG slice by one word
  float* ks = smem;                                // [kTokChunk][kstride]
  float* vs = ks + kTokChunk * kstride;            // [kTokChunk][rows_cta]
  float* as = vs + kTokChunk * rows_cta;           // [kTokChunk] alpha
  float* bs = as + kTokChunk;                      // [kTokChunk] beta

  const int rh = blockIdx.x;
  const int r = rh / H, h = rh % H;
  const int row0 = blockIdx.y * rows_cta;
  const int tid = threadIdx.x;
  const int lrow = tid / TPR, lt = tid % TPR;
  const int i = row0 + lrow;
  const bool active = i < d_v;

  float S[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) S[c] = 0.f;

  for (int p0 = 0; p0 < P; p0 += kTokChunk) {
    const int np = min(kTokChunk, P - p0);
    __syncthreads();
    for (int idx = tid; idx < np * d_k; idx += kPrefillThreads) {
      const int tp = idx / d_k, e = idx % d_k;
      const size_t src = ((size_t(r) * P + p0 + tp) * H + h) * size_t(d_k) + e;
      ks[tp * kstride + (e / SEG) * (SEG + 1) + (e % SEG)] = ld_in<TIn>(kp, src);
    }
    for (int idx = tid; idx < np * rows_cta; idx += kPrefillThreads) {
      const int tp = idx / rows_cta, rr = idx % rows_cta;
      const int ii = row0 + rr;
      float val = 0.f;
      if (ii < d_v) val = ld_in<TIn>(vp, ((size_t(r) * P + p0 + tp) * H + h) * size_t(d_v) + ii);
      vs[tp * rows_cta + rr] = val;
    }
    if (tid < np) {
      const size_t sidx = (size_t(r) * P + p0 + tid) * H + h;
      as[tid] = expf(gp[sidx]);
      bs[tid] = bp[sidx];
    }
    __syncthreads();
    for (int tp = 0; tp < np; ++tp) {
      const float* kk = ks + tp * kstride + lt * (SEG + 1);
      float u = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (c < SEG) u = fmaf(S[c], kk[c], u);
      u = group_sum(u, TPR);
      const float alpha = as[tp], beta = bs[tp];
      const float w = beta * (vs[tp * rows_cta + lrow] - alpha * u);
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (c < SEG) S[c] = fmaf(alpha, S[c], w * kk[c]);
    }
  }
  if (active) {
    float* dst = S_out + ((size_t(r) * H + h) * d_v + i) * size_t(d_k) + lt * SEG;
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if (c < SEG) dst[c] = S[c];
  }
}

cudaError_t launch_prefill(int R, int H, int d_k, int d_v, int P, int in_dtype, const void* k,
                           const void* v, const float* g, const float* beta, float* S_out,
                           cudaStream_t stream) {
  const int SEG = d_k < 32 ? d_k : 32;
  const int TPR = d_k / SEG;
  const int rows_cta = kPrefillThreads / TPR;
  const size_t smem =
      sizeof(float) * (kTokChunk * (d_k + TPR) + kTokChunk * rows_cta + 2 * kTokChunk);
  dim3 grid(R * H, (d_v + rows_cta - 1) / rows_cta);
  if (in_dtype == OLA_BF16)
    prefill_kernel<__nv_bfloat16><<<grid, kPrefillThreads, smem, stream>>>(
        R, H, d_k, d_v, P, k, v, g, beta, S_out);
  else
    prefill_kernel<float><<<grid, kPrefillThreads, smem, stream>>>(R, H, d_k, d_v, P, k, v, g,
                                                                   beta, S_out);
  return cudaGetLastError();
}

}  // namespace ola
