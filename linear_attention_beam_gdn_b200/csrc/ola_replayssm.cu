// History-replay decode step (the "ReplaySSM" comparison path): no per-beam state is stored,
// and every step rebuilds each beam's state from the shared state by replaying its decoded
// history.
//
// The OneLA listing's Abstract (arXiv) names two existing practices for large-beam
// linear-attention decoding: materialise a full recurrent state for every beam (the FullState
// path, ola_fullstate.cu) or repeatedly replay the shared history. "Scientific Impact
// Assessment: OneLA", §2 Methodological Rigor, lists the corresponding serving baselines
// (FullState, ReplaySSM). The pages describe the second practice only by that clause; the
// reading implemented here is its plainest form: each beam keeps the raw token inputs of its
// decode steps (k_j, v_j, alpha_j, beta_j, appended once per step and never moved, addressed
// through the same chain rows as the replay path), and at step t the state of new beam b with
// parent p is recomputed from S_ctx by applying the gated delta rule to the tokens on p's
// chain, j = 1..t-1, and then to b's own token:
//     S <- alpha_j S (I - beta_j k_j k_j^T) + beta_j v_j k_j^T      (row i: u_i = S_i . k_j,
//          S_i <- alpha_j S_i + beta_j (v_j[i] - alpha_j u_i) k_j)
//     o_t = S q_t.
// Row i of the state evolves independently of the others, so the state is never materialised
// in memory: it lives in registers, a row split over LPR lanes, as a scale sigma times a row
// S^ (S = sigma S^): a transition is then sigma <- alpha sigma, S^ += (w / sigma) k, one fused
// multiply-add per element instead of a multiply and a fused multiply-add (S^ is rescaled into
// S whenever sigma falls below 2^-60, so it stays far from fp32 overflow). The keys and values of
// the history are kept in the input dtype: the rebuilds stream the keys through L1/L2 for every
// beam, so their bytes, not the conversion, set the pace (measured: fp32 keys made the stress
// decode 1.3x slower).
//
// Grid: (request, head) x blocks of state rows. A CTA of 8 warps holds its rows of S_ctx in
// shared memory (read from HBM once per step and CTA) and walks every beam of the request,
// grouped by parent (a counting sort of the parents); each warp owns RPW rows and rebuilds
// them over the parent's chain once per parent, reading the chain's keys through L2 one
// ancestor ahead, keeps that state in shared memory and applies each child's own token to it.
// Nothing survives the step. fp32 arithmetic on CUDA cores throughout.
#include "ola_device.cuh"

namespace ola {

constexpr int kRsWarps = 8;
constexpr int kRsThreads = kRsWarps * 32;

template <int DK>
struct RsShape {
  static constexpr int LPR = DK >= 32 ? DK / 32 : 1;   // lanes per state row
  static constexpr int EL = DK / LPR;                  // columns per lane (32, or 16 at DK 16)
  static constexpr int RPW = 32 / LPR;                 // rows per warp
  static constexpr int ROWS = kRsWarps * RPW;          // rows per CTA
  static constexpr int V4 = EL / 4;                    // float4 per lane
};

// shared memory: S_ctx slices and the rebuilt parent state ([V4][kRsThreads] float4 each), then
// the beams grouped by parent and the counts of the sort ([B] int each)
template <int DK>
__host__ __device__ constexpr size_t rs_state_bytes() {
  return size_t(kRsThreads) * RsShape<DK>::EL * 4;
}
template <int DK>
__host__ __device__ constexpr size_t rs_smem_bytes(int B) {
  return 2 * rs_state_bytes<DK>() + 2 * size_t(B) * 4;
}

// EL consecutive inputs starting at element `e0` of row `row` of a [.., DK] array, widened
// to fp32.
template <typename TIn, int EL>
__device__ __forceinline__ void load_slice(float (&x)[EL], const void* base, size_t row, int e0,
                                           int DK) {
  if constexpr (sizeof(TIn) == 4) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) +
                                                      row * DK + e0);
#pragma unroll
    for (int j = 0; j < EL / 4; ++j) {
      const float4 f = __ldg(p + j);
      x[4 * j] = f.x;
      x[4 * j + 1] = f.y;
      x[4 * j + 2] = f.z;
      x[4 * j + 3] = f.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) +
                                                    row * DK + e0);
#pragma unroll
    for (int j = 0; j < EL / 8; ++j) {
      const uint4 u = __ldg(p + j);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        x[8 * j + 2 * m] = __uint_as_float(w[m] << 16);
        x[8 * j + 2 * m + 1] = __uint_as_float(w[m] & 0xffff0000u);
      }
    }
  }
}

// Parent of beam b as the append pass reads it (out of range: 0; the append pass reports it).
__device__ __forceinline__ int clamped_parent(const StepArgs& a, int r, int b) {
  const int p = a.parent[size_t(r) * a.B + b];
  return ((a.t == 1 && p != 0) || p < 0 || p >= a.B) ? 0 : p;
}

// One transition of the lane's slice of row i, the row held as sigma * S^:
// u = sigma (S^_i . k) (over the LPR lanes of the row), w = beta (v_i - alpha u),
// S_i <- alpha S_i + w k, i.e. sigma <- alpha sigma, S^_i += (w / sigma) k.
template <int EL, int LPR>
__device__ __forceinline__ void rs_transition(float (&S)[EL], float& sigma, const float (&k)[EL],
                                              float vi, float alpha, float beta) {
  float u = 0.f;
#pragma unroll
  for (int e = 0; e < EL; ++e) u = fmaf(S[e], k[e], u);
#pragma unroll
  for (int off = LPR >> 1; off > 0; off >>= 1) u += __shfl_xor_sync(0xffffffffu, u, off);
  const float w = beta * (vi - alpha * (sigma * u));
  sigma *= alpha;
  if (sigma < 0x1p-60f) {             // same for every lane (one beam's chain): no divergence
#pragma unroll
    for (int e = 0; e < EL; ++e) S[e] *= sigma;
    sigma = 1.f;
  }
  const float c = w / sigma;
#pragma unroll
  for (int e = 0; e < EL; ++e) S[e] = fmaf(c, k[e], S[e]);
}

template <typename TIn, int DK>
__global__ void __launch_bounds__(kRsThreads, 2)
replayssm_kernel(StepArgs a) {
  using Sh = RsShape<DK>;
  constexpr int LPR = Sh::LPR, EL = Sh::EL, RPW = Sh::RPW, ROWS = Sh::ROWS, V4 = Sh::V4;
  static_assert(EL % 8 == 0, "a lane's slice is whole 16-byte vectors");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float4* S0 = reinterpret_cast<float4*>(smem_raw);      // [V4][kRsThreads]: S_ctx slices
  float4* SP = S0 + V4 * kRsThreads;                     // the rebuilt state of the current parent
  int* ord = reinterpret_cast<int*>(SP + V4 * kRsThreads);   // [B] beams grouped by parent
  int* cnt = ord + a.B;                                       // [B] counts, then offsets

  const int rh = blockIdx.x;
  const int r = rh / a.H, h = rh % a.H;
  const int row_base = blockIdx.y * ROWS;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int part = lane % LPR;
  const int row = row_base + warp * RPW + lane / LPR;
  const bool row_ok = row < a.d_v;
  const int e0 = part * EL;
  const int t = a.t, n_anc = t - 1;

  // 1. this CTA's rows of S_ctx -> shared memory, interleaved so that every access is one
  //    16-byte vector per lane, consecutive lanes on consecutive vectors
  {
    const float* src = a.S + (size_t(r) * a.H + h) * size_t(a.d_v) * DK;
#pragma unroll
    for (int j = 0; j < V4; ++j) {
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      if (row_ok) f = __ldg(reinterpret_cast<const float4*>(src + size_t(row) * DK + e0) + j);
      S0[j * kRsThreads + tid] = f;
    }
  }

  // 2. append this step's tokens (slot t-1) and the chain rows: the first row block only
  if (blockIdx.y == 0) {
    const int slot = t - 1;
    for (int b = warp; b < a.B; b += kRsWarps) {
      const size_t in = (size_t(r) * a.B + b) * a.H + h;
      const size_t rec = rec_index(a, slot, r, h, b);
      for (int e = lane; e < DK; e += 32)
        static_cast<TIn*>(a.Kr)[rec * DK + e] = static_cast<const TIn*>(a.k)[in * DK + e];
      for (int e = lane; e < a.d_v; e += 32)
        static_cast<TIn*>(a.Vr)[rec * a.d_v + e] =
            static_cast<const TIn*>(a.v)[in * size_t(a.d_v) + e];
      if (lane == 0) {
        a.A[rec] = expf(a.g[in]);
        a.Br[rec] = a.beta[in];
      }
      if (h == 0) {
        const int p = checked_parent(a, r, b);
        if (lane < t) {
          int val = b;
          if (lane < n_anc) val = a.C[chain_row(a, t - 2, r, p) + lane];
          a.C[chain_row(a, t - 1, r, b) + lane] = val;
        }
      }
    }
  }
  // 3. the beams grouped by parent: a counting sort of the (clamped) parents; the order within
  //    a group does not matter (every child of a parent starts from the same rebuilt state)
  for (int b = tid; b < a.B; b += kRsThreads) cnt[b] = 0;
  __syncthreads();
  for (int b = tid; b < a.B; b += kRsThreads) atomicAdd(&cnt[clamped_parent(a, r, b)], 1);
  __syncthreads();
  if (warp == 0) {                                       // exclusive scan of the counts
    int carry = 0;
    for (int base = 0; base < a.B; base += 32) {
      const int x = base + lane < a.B ? cnt[base + lane] : 0;
      int y = x;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int z = __shfl_up_sync(0xffffffffu, y, off);
        if (lane >= off) y += z;
      }
      if (base + lane < a.B) cnt[base + lane] = carry + y - x;
      carry += __shfl_sync(0xffffffffu, y, 31);
    }
  }
  __syncthreads();
  for (int b = tid; b < a.B; b += kRsThreads) ord[atomicAdd(&cnt[clamped_parent(a, r, b)], 1)] = b;
  __syncthreads();

  // 4. every beam of the request, a parent's children in a row: rebuild this warp's rows from
  //    S_ctx along the parent's chain once per parent (kept in SP), apply the beam's own token,
  //    project onto q_t
  int prev_p = -1;
  float sigma_p = 1.f;
  for (int ib = 0; ib < a.B; ++ib) {
    const int b = ord[ib];
    const int p = clamped_parent(a, r, b);
    float S[EL];
    float kc[EL], kn[EL];
    float vc = 0.f, ac = 1.f, bc = 0.f, sigma = 1.f;
    const size_t in = (size_t(r) * a.B + b) * a.H + h;
    if (p != prev_p) {
      // the parent's state: S_ctx, then the tokens of its chain
      int cidx = 0;
      if (lane < n_anc) cidx = __ldg(a.C + chain_row(a, t - 2, r, p) + lane);
#pragma unroll
      for (int j = 0; j < V4; ++j) {
        const float4 f = S0[j * kRsThreads + tid];
        S[4 * j] = f.x;
        S[4 * j + 1] = f.y;
        S[4 * j + 2] = f.z;
        S[4 * j + 3] = f.w;
      }
      auto fetch = [&](int j, float (&kx)[EL], float& vx, float& ax, float& bx) {
        const int c = __shfl_sync(0xffffffffu, cidx, j);
        const size_t rec = rec_index(a, j, r, h, c);
        load_slice<TIn, EL>(kx, a.Kr, rec, e0, DK);
        vx = row_ok ? to_f32(static_cast<const TIn*>(a.Vr)[rec * a.d_v + row]) : 0.f;
        ax = __ldg(a.A + rec);
        bx = __ldg(a.Br + rec);
      };
      if (n_anc > 0) fetch(0, kc, vc, ac, bc);
      for (int j = 0; j < n_anc; ++j) {
        float vn = 0.f, an = 1.f, bn = 0.f;
        if (j + 1 < n_anc) fetch(j + 1, kn, vn, an, bn);   // one position ahead
        rs_transition<EL, LPR>(S, sigma, kc, vc, ac, bc);
        if (j + 1 < n_anc) {
#pragma unroll
          for (int e = 0; e < EL; ++e) kc[e] = kn[e];
          vc = vn;
          ac = an;
          bc = bn;
        }
      }
#pragma unroll
      for (int j = 0; j < V4; ++j)
        SP[j * kRsThreads + tid] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
      sigma_p = sigma;
      prev_p = p;
    } else {
#pragma unroll
      for (int j = 0; j < V4; ++j) {
        const float4 f = SP[j * kRsThreads + tid];
        S[4 * j] = f.x;
        S[4 * j + 1] = f.y;
        S[4 * j + 2] = f.z;
        S[4 * j + 3] = f.w;
      }
      sigma = sigma_p;
    }
    // the beam's own token
    load_slice<TIn, EL>(kc, a.k, in, e0, DK);
    vc = row_ok ? to_f32(static_cast<const TIn*>(a.v)[in * size_t(a.d_v) + row]) : 0.f;
    ac = expf(__ldg(a.g + in));
    bc = __ldg(a.beta + in);
    rs_transition<EL, LPR>(S, sigma, kc, vc, ac, bc);
    // o_t[i] = S_i . q_t
    load_slice<TIn, EL>(kc, a.q, in, e0, DK);
    float o = 0.f;
#pragma unroll
    for (int e = 0; e < EL; ++e) o = fmaf(S[e], kc[e], o);
#pragma unroll
    for (int off = LPR >> 1; off > 0; off >>= 1) o += __shfl_xor_sync(0xffffffffu, o, off);
    if (row_ok && part == 0) a.o[in * size_t(a.d_v) + row] = sigma * o;
  }
}

template <typename TIn, int DK>
static cudaError_t launch_rs_dk(const StepArgs& a, cudaStream_t stream) {
  using Sh = RsShape<DK>;
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = once_per_device(configured, [] {
    return cudaFuncSetAttribute(replayssm_kernel<TIn, DK>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(rs_smem_bytes<DK>(4096)));
  });
  if (e != cudaSuccess) return e;
  const dim3 grid(unsigned(a.R) * a.H, unsigned((a.d_v + Sh::ROWS - 1) / Sh::ROWS));
  replayssm_kernel<TIn, DK><<<grid, kRsThreads, rs_smem_bytes<DK>(a.B), stream>>>(a);
  return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_rs_t(const StepArgs& a, cudaStream_t stream) {
  switch (a.d_k) {
    case 16: return launch_rs_dk<TIn, 16>(a, stream);
    case 32: return launch_rs_dk<TIn, 32>(a, stream);
    case 64: return launch_rs_dk<TIn, 64>(a, stream);
    case 128: return launch_rs_dk<TIn, 128>(a, stream);
    case 256: return launch_rs_dk<TIn, 256>(a, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_replayssm(const StepArgs& a, int in_dtype, cudaStream_t stream) {
  return in_dtype == OLA_BF16 ? launch_rs_t<__nv_bfloat16>(a, stream)
                              : launch_rs_t<float>(a, stream);
}

}  // namespace ola
