// FullState decode step: one materialised d_v x d_k fp32 state per (request, beam, head).
//
// The OneLA listing's Abstract (arXiv) names this as the practice of existing linear-attention
// servers: a full recurrent state for every beam. "Scientific Impact Assessment: OneLA",
// §2 Methodological Rigor, describes the controlled FullState baseline that runs the same
// decode pipeline with this representation. Here it is an in-library comparison path.
//
// Per new beam b with parent p: S_p is the parent's state (the shared state at step 1),
//     u = S_p k,  w = beta (v - alpha u),  S_b = alpha S_p + w k^T,  o = S_b q.
// One pass over HBM: each row of S_p is read once, S_b's row is written once. TPR threads
// hold one row (VPT float4 each) and combine the two row dot products with shuffles.
#include "ola_device.cuh"

namespace ola {

constexpr int kFsThreads = 256;

template <typename TIn, int DK>
__global__ void __launch_bounds__(kFsThreads)
fullstate_kernel(StepArgs a) {
  constexpr int TPR = DK / 4 < 32 ? DK / 4 : 32;   // threads per row
  constexpr int VPT = DK / (4 * TPR);              // float4 per thread per row
  constexpr int RPP = kFsThreads / TPR;            // rows per pass
  constexpr int UNR = 2;                           // rows in flight per thread

  const int bid = blockIdx.x;                      // (r, h, b), b fastest
  const int b = bid % a.B;
  const int rh = bid / a.B;
  const int h = rh % a.H, r = rh / a.H;
  const int tid = threadIdx.x;
  const int grp = tid / TPR, lt = tid % TPR;
  const int d_v = a.d_v;

  const int p = checked_parent(a, r, b);
  if (h == 0 && tid < a.t) {
    // ancestry row for ola_get_ancestry: parent's row ++ [b]
    int val = b;
    if (tid < a.t - 1) val = a.C[chain_row(a, a.t - 2, r, p) + tid];
    a.C[chain_row(a, a.t - 1, r, b) + tid] = val;
  }

  const size_t in_k = ((size_t(r) * a.B + b) * a.H + h) * DK;
  float4 kq[VPT], qq[VPT];
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int e = (j * TPR + lt) * 4;
    kq[j] = make_float4(ld_in<TIn>(a.k, in_k + e), ld_in<TIn>(a.k, in_k + e + 1),
                        ld_in<TIn>(a.k, in_k + e + 2), ld_in<TIn>(a.k, in_k + e + 3));
    qq[j] = make_float4(ld_in<TIn>(a.q, in_k + e), ld_in<TIn>(a.q, in_k + e + 1),
                        ld_in<TIn>(a.q, in_k + e + 2), ld_in<TIn>(a.q, in_k + e + 3));
  }
  const size_t sidx = (size_t(r) * a.B + b) * a.H + h;
  const float alpha = expf(a.g[sidx]);
  const float beta = a.beta[sidx];
  const size_t in_v = sidx * size_t(d_v);

  const float* src = (a.t == 1) ? a.S + (size_t(r) * a.H + h) * size_t(d_v) * DK
                                : a.FS_prev + ((size_t(r) * a.H + h) * a.B + p) * size_t(d_v) * DK;
  float* dst = a.FS_cur + ((size_t(r) * a.H + h) * a.B + b) * size_t(d_v) * DK;

  for (int row0 = 0; row0 < d_v; row0 += RPP * UNR) {
    float4 s[UNR][VPT];
#pragma unroll
    for (int uu = 0; uu < UNR; ++uu) {
      const int i = row0 + uu * RPP + grp;
#pragma unroll
      for (int j = 0; j < VPT; ++j)
        s[uu][j] = (i < d_v) ? __ldcs(reinterpret_cast<const float4*>(src + size_t(i) * DK) +
                                      j * TPR + lt)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int uu = 0; uu < UNR; ++uu) {
      const int i = row0 + uu * RPP + grp;
      float u = 0.f;
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        u = fmaf(s[uu][j].x, kq[j].x, u);
        u = fmaf(s[uu][j].y, kq[j].y, u);
        u = fmaf(s[uu][j].z, kq[j].z, u);
        u = fmaf(s[uu][j].w, kq[j].w, u);
      }
      u = group_sum(u, TPR);
      const float vi = (i < d_v) ? ld_in<TIn>(a.v, in_v + i) : 0.f;
      const float w = beta * (vi - alpha * u);
      float od = 0.f;
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        float4 n;
        n.x = fmaf(alpha, s[uu][j].x, w * kq[j].x);
        n.y = fmaf(alpha, s[uu][j].y, w * kq[j].y);
        n.z = fmaf(alpha, s[uu][j].z, w * kq[j].z);
        n.w = fmaf(alpha, s[uu][j].w, w * kq[j].w);
        od = fmaf(n.x, qq[j].x, od);
        od = fmaf(n.y, qq[j].y, od);
        od = fmaf(n.z, qq[j].z, od);
        od = fmaf(n.w, qq[j].w, od);
        if (i < d_v) __stcs(reinterpret_cast<float4*>(dst + size_t(i) * DK) + j * TPR + lt, n);
      }
      od = group_sum(od, TPR);
      if (i < d_v && lt == 0) a.o[in_v + i] = od;
    }
  }
}

template <typename TIn>
static cudaError_t launch_fs_t(const StepArgs& a, cudaStream_t stream) {
  const unsigned grid = unsigned(a.R) * a.H * a.B;
  switch (a.d_k) {
    case 16: fullstate_kernel<TIn, 16><<<grid, kFsThreads, 0, stream>>>(a); break;
    case 32: fullstate_kernel<TIn, 32><<<grid, kFsThreads, 0, stream>>>(a); break;
    case 64: fullstate_kernel<TIn, 64><<<grid, kFsThreads, 0, stream>>>(a); break;
    case 128: fullstate_kernel<TIn, 128><<<grid, kFsThreads, 0, stream>>>(a); break;
    case 256: fullstate_kernel<TIn, 256><<<grid, kFsThreads, 0, stream>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_fullstate(const StepArgs& a, int in_dtype, cudaStream_t stream) {
  return in_dtype == OLA_BF16 ? launch_fs_t<__nv_bfloat16>(a, stream)
                              : launch_fs_t<float>(a, stream);
}

}  // namespace ola
