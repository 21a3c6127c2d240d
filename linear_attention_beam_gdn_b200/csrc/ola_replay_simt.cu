// Projection-replay decode step, CUDA-core fp32 path.
//
// "Scientific Impact Assessment: OneLA", §1 Core Contribution and Additional Observations: a
// GDN layer meets its prior state only through the key and query contractions, so a beam's
// state never has to be rebuilt; each beam keeps append-only transition records of
// O(d_v + d_k). For new beam b (parent p, chain of records j = 1..t-1):
//     S_{t-1} x = (prod_j alpha_j) S_ctx x + sum_j (prod_{i>j} alpha_i) w_j (k_j . x)
//     u = S_{t-1} k_t,  w_t = beta_t (v_t - alpha_t u),  o_t = alpha_t S_{t-1} q_t + (k_t . q_t) w_t
// and the record (w_t, k_t, alpha_t) is appended at slot t-1 without touching older records
// (the OneLA listing's Abstract: beams are updated without moving or copying records).
//
// One CTA handles one (request, head) and a chunk of NB beams:
//   1. [q; k] of the chunk -> shared memory (fp32);
//   2. Y = S_ctx [q k] on CUDA cores (each thread: one row of S_ctx, 2 NB / (256 / d_v)
//      columns), the shared state read once per chunk through L1/L2;
//   3. per beam (one warp): chain lookup, suffix products of the chain's alphas, the dot
//      products k_j . k_t and k_j . q_t, and the append of k_t, alpha_t and the chain row;
//   4. per (beam, row): u, w_t, o_t from Y and the ancestors' w_j, then stores of o and w_t.
#include "ola_device.cuh"

namespace ola {

constexpr int kSimtThreads = 256;

struct SimtLayout {
  int NB, TA;
  size_t x_off, y_off, cu_off, cq_off, rec_off, sc_off, bytes;
};

__host__ __device__ inline SimtLayout simt_layout(int d_k, int d_v, int T_max) {
  SimtLayout L;
  L.NB = 2048 / d_v;
  if (L.NB > 64) L.NB = 64;
  L.TA = T_max > 1 ? T_max - 1 : 1;
  L.x_off = 0;
  L.y_off = L.x_off + sizeof(float) * 2 * L.NB * d_k;
  L.cu_off = L.y_off + sizeof(float) * 2 * L.NB * d_v;
  L.cq_off = L.cu_off + sizeof(float) * L.NB * L.TA;
  L.rec_off = L.cq_off + sizeof(float) * L.NB * L.TA;
  L.sc_off = L.rec_off + sizeof(int) * L.NB * L.TA;
  L.bytes = L.sc_off + sizeof(float) * 4 * L.NB;
  return L;
}

template <typename TIn>
__global__ void __launch_bounds__(kSimtThreads)
replay_simt_kernel(StepArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int d_k = a.d_k, d_v = a.d_v;
  const SimtLayout L = simt_layout(d_k, d_v, a.T_max);
  const int NB = L.NB, TA = L.TA;
  float* X = reinterpret_cast<float*>(smem_raw + L.x_off);     // [2NB][d_k]: q rows, k rows
  float* Y = reinterpret_cast<float*>(smem_raw + L.y_off);     // [2NB][d_v]
  float* cu = reinterpret_cast<float*>(smem_raw + L.cu_off);   // [NB][TA]
  float* cq = reinterpret_cast<float*>(smem_raw + L.cq_off);   // [NB][TA]
  int* rec = reinterpret_cast<int*>(smem_raw + L.rec_off);     // [NB][TA]
  float* sc = reinterpret_cast<float*>(smem_raw + L.sc_off);   // [NB][4]: ep, alpha, beta, c0

  const int n_chunks = (a.B + NB - 1) / NB;
  const int chunk = blockIdx.x % n_chunks;
  const int rh = blockIdx.x / n_chunks;
  const int r = rh / a.H, h = rh % a.H;
  const int b0 = chunk * NB;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = a.t, n_anc = t - 1;

  // 1. stage q, k of the chunk
  for (int idx = tid; idx < 2 * NB * d_k; idx += kSimtThreads) {
    const int c = idx / d_k, e = idx % d_k;
    const int b = b0 + (c % NB);
    float val = 0.f;
    if (b < a.B) {
      const size_t src = ((size_t(r) * a.B + b) * a.H + h) * size_t(d_k) + e;
      val = (c < NB) ? ld_in<TIn>(a.q, src) : ld_in<TIn>(a.k, src);
    }
    X[idx] = val;
  }
  __syncthreads();

  // 2. Y[c][i] = sum_e S_ctx[i][e] X[c][e]
  {
    const int n_cg = kSimtThreads / d_v;         // threads per row (d_v <= 256)
    const int i = tid % d_v, cg = tid / d_v;
    const int cpt = 2 * NB / n_cg;               // columns per thread (<= 16)
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    const float4* srow =
        reinterpret_cast<const float4*>(a.S + ((size_t(r) * a.H + h) * d_v + i) * size_t(d_k));
    for (int e4 = 0; e4 < d_k / 4; ++e4) {
      const float4 s = __ldg(srow + e4);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (j < cpt) {
          const float4 x = reinterpret_cast<const float4*>(X + (cg + j * n_cg) * d_k)[e4];
          acc[j] = fmaf(s.x, x.x, acc[j]);
          acc[j] = fmaf(s.y, x.y, acc[j]);
          acc[j] = fmaf(s.z, x.z, acc[j]);
          acc[j] = fmaf(s.w, x.w, acc[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < cpt) Y[(cg + j * n_cg) * d_v + i] = acc[j];
  }

  // 3. per-beam scalars: one warp per beam
  for (int bl = warp; bl < NB; bl += kSimtThreads / 32) {
    const int b = b0 + bl;
    if (b >= a.B) continue;
    const int p = checked_parent(a, r, b);
    int my_rec = 0;
    float my_alpha = 1.f;
    if (lane < n_anc) {
      my_rec = a.C[chain_row(a, t - 2, r, p) + lane];
      my_alpha = a.A[rec_index(a, lane, r, h, my_rec)];
    }
    // inclusive suffix product over the chain: x_s = prod_{i >= s} alpha_i
    float x = my_alpha;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_down_sync(0xffffffffu, x, off);
      if (lane + off < 32) x *= y;
    }
    const float ep = __shfl_sync(0xffffffffu, x, 0);           // prod of all chain alphas
    const float dec = __shfl_down_sync(0xffffffffu, x, 1);     // prod_{i > s} alpha_i
    const float* xq = X + bl * d_k;
    const float* xk = X + (NB + bl) * d_k;
    for (int s = 0; s < n_anc; ++s) {
      const int rs = __shfl_sync(0xffffffffu, my_rec, s);
      const size_t kb = rec_index(a, s, r, h, rs) * size_t(d_k);
      float dk = 0.f, dq = 0.f;
      for (int e = lane; e < d_k; e += 32) {
        const float kj = ld_in<TIn>(a.Kr, kb + e);
        dk = fmaf(kj, xk[e], dk);
        dq = fmaf(kj, xq[e], dq);
      }
      dk = warp_sum(dk);
      dq = warp_sum(dq);
      if (lane == s) {
        cu[bl * TA + s] = dec * dk;
        cq[bl * TA + s] = dec * dq;
        rec[bl * TA + s] = rs;
      }
    }
    float c0 = 0.f;
    for (int e = lane; e < d_k; e += 32) c0 = fmaf(xk[e], xq[e], c0);
    c0 = warp_sum(c0);
    const size_t sidx = (size_t(r) * a.B + b) * a.H + h;
    const float alpha = expf(a.g[sidx]);
    if (lane == 0) {
      sc[bl * 4 + 0] = ep;
      sc[bl * 4 + 1] = alpha;
      sc[bl * 4 + 2] = a.beta[sidx];
      sc[bl * 4 + 3] = c0;
      a.A[rec_index(a, t - 1, r, h, b)] = alpha;
    }
    // append k_t (bit copy of the input) and, once per request, the chain row
    const size_t kdst = rec_index(a, t - 1, r, h, b) * size_t(d_k);
    const size_t ksrc = sidx * size_t(d_k);
    for (int e = lane; e < d_k; e += 32)
      static_cast<TIn*>(a.Kr)[kdst + e] = static_cast<const TIn*>(a.k)[ksrc + e];
    if (h == 0 && lane < t) a.C[chain_row(a, t - 1, r, b) + lane] = (lane < n_anc) ? my_rec : b;
  }
  __syncthreads();

  // 4. per (beam, row): u, w_t, o_t
  {
    const int n_bg = kSimtThreads / d_v;
    const int i = tid % d_v, bg = tid / d_v;
    for (int bl = bg; bl < NB; bl += n_bg) {
      const int b = b0 + bl;
      if (b >= a.B) break;
      const float ep = sc[bl * 4 + 0], alpha = sc[bl * 4 + 1], beta = sc[bl * 4 + 2],
                  c0 = sc[bl * 4 + 3];
      float u = ep * Y[(NB + bl) * d_v + i];
      float qa = ep * Y[bl * d_v + i];
      for (int s = 0; s < n_anc; ++s) {
        const float wv = __ldg(a.W + rec_index(a, s, r, h, rec[bl * TA + s]) * size_t(d_v) + i);
        u = fmaf(cu[bl * TA + s], wv, u);
        qa = fmaf(cq[bl * TA + s], wv, qa);
      }
      const size_t sidx = (size_t(r) * a.B + b) * a.H + h;
      const float vi = ld_in<TIn>(a.v, sidx * size_t(d_v) + i);
      const float w = beta * (vi - alpha * u);
      a.o[sidx * size_t(d_v) + i] = fmaf(alpha, qa, c0 * w);
      a.W[rec_index(a, t - 1, r, h, b) * size_t(d_v) + i] = w;
    }
  }
}

size_t replay_simt_smem(int d_k, int d_v, int T_max) {
  return simt_layout(d_k, d_v, T_max).bytes;
}

cudaError_t launch_replay_simt(const StepArgs& a, int in_dtype, cudaStream_t stream) {
  const SimtLayout L = simt_layout(a.d_k, a.d_v, a.T_max);
  const int n_chunks = (a.B + L.NB - 1) / L.NB;
  const unsigned grid = unsigned(a.R) * a.H * n_chunks;
  if (in_dtype == OLA_BF16) {
    cudaFuncSetAttribute(replay_simt_kernel<__nv_bfloat16>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(L.bytes));
    replay_simt_kernel<__nv_bfloat16><<<grid, kSimtThreads, L.bytes, stream>>>(a);
  } else {
    cudaFuncSetAttribute(replay_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         int(L.bytes));
    replay_simt_kernel<float><<<grid, kSimtThreads, L.bytes, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace ola
