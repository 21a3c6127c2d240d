// Record reclamation: folding the shared prefix of the beams' ancestry into the shared state.
//
// "Scientific Impact Assessment: OneLA", §1 Core Contribution: every beam is the shared
// post-prefill state plus the append-only transition records along its chain, and the
// parent-pointer ancestry index handles pruning. Once pruning has left every live beam of a
// request with the same records at the oldest chain slots (beam search converges), those
// records no longer distinguish any beam: applying them to the shared state,
//     S <- alpha_j S + w_j k_j^T        for each shared record j, oldest first
// (the gated delta rule written with the record: alpha S (I - beta k k^T) + beta v k^T =
// alpha S + beta (v - alpha S k) k^T = alpha S + w k^T), gives a shared state from which the
// remaining records replay to the same outputs, and their step slots can be reused. The fold
// covers the slots shared by every request of the handle, so that all requests keep one step
// counter.
#include "ola_device.cuh"

namespace ola {

// Length of the chain prefix shared by all beams of request r: the first chain slot s < t - 1
// at which two beams differ (t - 1 if none), over the chain rows of the current step.
__global__ void __launch_bounds__(256) common_prefix_kernel(const int* __restrict__ C, int R, int B,
                                                           int T_max, int t, int* __restrict__ out) {
  const int r = blockIdx.x;
  __shared__ int differs;
  const int* rows = C + (size_t(t - 1) * R + r) * size_t(B) * T_max;   // [B][T_max]
  int c = t - 1;
  for (int s = 0; s < t - 1; ++s) {
    if (threadIdx.x == 0) differs = 0;
    __syncthreads();
    const int ref = rows[s];
    for (int b = threadIdx.x; b < B; b += blockDim.x)
      if (rows[size_t(b) * T_max + s] != ref) differs = 1;
    __syncthreads();
    const int d = differs;
    __syncthreads();
    if (d) {
      c = s;
      break;
    }
  }
  if (threadIdx.x == 0) out[r] = c;
}

// S[r][h] <- alpha_j S + w_j k_j^T for the records j of chain slots 0..c-1 (taken from beam 0's
// chain: every beam shares them). One thread per state row.
//   layout 0: records [T_max][R][H][B], w fp32 [d_v]
//   layout 1: records [T_max][R][B][H], w as bf16 hi and lo planes [2][d_v]
//   layout 2: records [T_max][R][H][B] holding the raw token (history-replay path): k and v
//             in the input dtype, and beta; w_j[i] = beta_j (v_j[i] - alpha_j S_i . k_j) is formed
//             from the state folded so far (the gated delta rule itself)
template <typename TK>
__global__ void __launch_bounds__(128) fold_kernel(float* __restrict__ S, const void* __restrict__ Wp,
                                                  const TK* __restrict__ Kr,
                                                  const float* __restrict__ A,
                                                  const float* __restrict__ Bt,
                                                  const int* __restrict__ C, int R, int H,
                                                  int d_k, int d_v, int B, int T_max, int t,
                                                  int c, int layout) {
  const size_t row = blockIdx.x * size_t(blockDim.x) + threadIdx.x;    // (r, h, i)
  if (row >= size_t(R) * H * d_v) return;
  const int i = int(row % d_v);
  const int h = int((row / d_v) % H);
  const int r = int(row / (size_t(d_v) * H));
  float* Srow = S + row * d_k;
  const int* chain = C + (size_t(t - 1) * R + r) * size_t(B) * T_max;   // beam 0's chain
  for (int s = 0; s < c; ++s) {
    const int b = chain[s];
    const size_t rec = layout != 1 ? ((size_t(s) * R + r) * H + h) * size_t(B) + b
                                   : ((size_t(s) * R + r) * B + b) * size_t(H) + h;
    const float al = A[rec];
    const TK* k = Kr + rec * d_k;
    float w;
    if (layout == 0) {
      w = static_cast<const float*>(Wp)[rec * d_v + i];
    } else if (layout == 1) {
      const __nv_bfloat16* wb = static_cast<const __nv_bfloat16*>(Wp) + rec * 2 * d_v;
      w = __bfloat162float(wb[i]) + __bfloat162float(wb[d_v + i]);
    } else {
      float u = 0.f;
      for (int x = 0; x < d_k; ++x) u = fmaf(Srow[x], float(k[x]), u);
      w = Bt[rec] * (float(static_cast<const TK*>(Wp)[rec * d_v + i]) - al * u);
    }
    for (int x = 0; x < d_k; ++x) Srow[x] = fmaf(al, Srow[x], w * float(k[x]));
  }
}

// Chain rows of the current step moved down by c slots: C[t-1-c][r][b][j] = C[t-1][r][b][j+c].
__global__ void chain_shift_kernel(int* __restrict__ C, int R, int B, int T_max, int t, int c) {
  const size_t rb = blockIdx.x * size_t(blockDim.x) + threadIdx.x;
  if (rb >= size_t(R) * B) return;
  const int* src = C + (size_t(t - 1) * R * B + rb) * T_max;
  int* dst = C + (size_t(t - 1 - c) * R * B + rb) * T_max;
  for (int j = 0; j + c < t; ++j) dst[j] = src[j + c];
}

cudaError_t launch_common_prefix(const int* C, int R, int B, int T_max, int t, int* out,
                                 cudaStream_t stream) {
  common_prefix_kernel<<<R, 256, 0, stream>>>(C, R, B, T_max, t, out);
  return cudaGetLastError();
}

cudaError_t launch_fold(float* S, const void* W, const void* Kr, int k_is_bf16, const float* A,
                        const float* Bt, const int* C, int R, int H, int d_k, int d_v, int B,
                        int T_max, int t, int c, int layout, cudaStream_t stream) {
  const size_t rows = size_t(R) * H * d_v;
  const unsigned grid = unsigned((rows + 127) / 128);
  if (k_is_bf16)
    fold_kernel<__nv_bfloat16><<<grid, 128, 0, stream>>>(
        S, W, static_cast<const __nv_bfloat16*>(Kr), A, Bt, C, R, H, d_k, d_v, B, T_max, t, c,
        layout);
  else
    fold_kernel<float><<<grid, 128, 0, stream>>>(S, W, static_cast<const float*>(Kr), A, Bt, C, R,
                                                 H, d_k, d_v, B, T_max, t, c, layout);
  return cudaGetLastError();
}

cudaError_t launch_chain_shift(int* C, int R, int B, int T_max, int t, int c,
                               cudaStream_t stream) {
  const size_t n = size_t(R) * B;
  chain_shift_kernel<<<unsigned((n + 255) / 256), 256, 0, stream>>>(C, R, B, T_max, t, c);
  return cudaGetLastError();
}

}  // namespace ola
