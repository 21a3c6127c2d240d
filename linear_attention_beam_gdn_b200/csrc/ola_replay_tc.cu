// Projection-replay decode step on the tcgen05 tensor cores (sm_100a).
//
// Same mathematics as the CUDA-core path ("Scientific Impact Assessment: OneLA", §1 Core
// Contribution: a shared post-prefill state, append-only transition records, projection
// replay through the key and query contractions, and one fused kernel that reuses the
// shared state across beams):
//     Y = S_ctx [q_b  k_b]_{b in chunk}                       (tensor cores)
//     u = e S_ctx k_t + sum_j c^k_j w_j,  w_t = beta (v_t - alpha u)
//     o_t = alpha (e S_ctx q_t + sum_j c^q_j w_j) + (k_t . q_t) w_t
// with e = prod of the chain's alphas and c^x_j = (prod_{i>j} alpha_i) (k_j . x).
//
// The only dense contraction is Y. S_ctx (fp32) is split once at create time into a bf16 high
// part and a bf16 remainder, S = S_hi + S_lo + O(2^-17 |S|), and both are multiplied by the
// bf16 q and k (exact inputs) into one fp32 accumulator in tensor memory.
//
// CTA = one (request, head) x a chunk of NB beams, 9 warps:
//   warp 8 lane 0 : TMA producer and MMA issuer. K is cut into 64-wide slices (one 128-byte
//                   swizzle atom); each slice stage holds S_hi, S_lo [M_pad x 64] and the
//                   chunk's [q; k] [2 NB x 64] (bf16, 128B swizzle), two stages in a ring.
//                   Per slice: 4 k-steps x M-tiles x (hi, lo) tcgen05.mma (M = 128,
//                   N = 2 NB, K = 16) into D [128 lanes x 2 NB columns] per M-tile.
//   warp 8        : allocates / frees the tensor memory.
//   warps 0..7    : while the MMAs run, one warp per beam does the chain lookup, the chain's
//                   alpha suffix products, k_j . k_t and k_j . q_t, and appends k_t, alpha_t
//                   and the chain row; then, once D is complete, each thread takes one row
//                   i of d_v (tensor-memory lane) for half of the chunk's beams (or one
//                   M-tile of a 256-wide d_v) and produces u, w_t, o_t with coalesced
//                   128-byte loads of the ancestors' w_j and stores of o and w_t.
// Every wait is bounded; on timeout the kernel records OLA_ERR_TIMEOUT and finishes.
#include "ola_device.cuh"

namespace ola {

constexpr int kTcThreads = 288;  // 8 epilogue warps + 1 control warp

template <int EPL> struct BfVec;
template <> struct BfVec<2> { using T = uint32_t; };
template <> struct BfVec<4> { using T = uint2; };
template <> struct BfVec<8> { using T = uint4; };

template <int EPL>
__device__ __forceinline__ void unpack_bf16(const typename BfVec<EPL>::T& raw, float (&f)[EPL]) {
  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int j = 0; j < EPL / 2; ++j) {
    const float2 x = __bfloat1622float2(h2[j]);
    f[2 * j] = x.x;
    f[2 * j + 1] = x.y;
  }
}

struct TcLayout {
  int MT, MROWS, NSL, NST, NB, TA;
  uint32_t a_bytes, x_bytes, stage_bytes, ncols;
  size_t bar_off, sc_off, cu_off, cq_off, rec_off, bytes;
};

__host__ __device__ inline TcLayout tc_layout(int d_k, int d_v, int NB, int T_max) {
  TcLayout L;
  L.MT = (d_v + 127) / 128;
  L.MROWS = L.MT * 128;
  L.NSL = d_k / 64;
  L.NST = L.NSL < 2 ? L.NSL : 2;
  L.NB = NB;
  L.TA = T_max > 1 ? T_max - 1 : 1;
  L.a_bytes = uint32_t(L.MROWS) * 128u;
  L.x_bytes = uint32_t(2 * NB) * 128u;
  L.stage_bytes = 2u * L.a_bytes + L.x_bytes;
  uint32_t need = uint32_t(L.MT * 2 * NB), c = 32;
  while (c < need) c <<= 1;
  L.ncols = c;
  L.bar_off = size_t(L.NST) * L.stage_bytes;            // full[2], empty[2], done, holder
  L.sc_off = L.bar_off + 64;
  L.cu_off = L.sc_off + sizeof(float) * 4 * NB;
  L.cq_off = L.cu_off + sizeof(float) * NB * L.TA;
  L.rec_off = L.cq_off + sizeof(float) * NB * L.TA;
  L.bytes = L.rec_off + sizeof(int) * NB * L.TA + 1024;  // + slack for 1024-B alignment
  return L;
}

template <int DK, int DV>
__global__ void __launch_bounds__(kTcThreads, DV <= 128 ? 2 : 1)
replay_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_shi,
                 const __grid_constant__ CUtensorMap tm_slo, StepArgs a, int NB) {
  constexpr int EPL = DK / 32;
  using Vec = typename BfVec<EPL>::T;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const TcLayout L = tc_layout(DK, DV, NB, a.T_max);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* empty = full + 2;
  uint64_t* done = full + 4;
  uint32_t* holder = reinterpret_cast<uint32_t*>(full + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + 6);
  float* sc = reinterpret_cast<float*>(smem + L.sc_off);        // [NB][4]: e, alpha, beta, c0
  float* cu = reinterpret_cast<float*>(smem + L.cu_off);        // [NB][TA]
  float* cq = reinterpret_cast<float*>(smem + L.cq_off);        // [NB][TA]
  int* rec = reinterpret_cast<int*>(smem + L.rec_off);          // [NB][TA]
  const int TA = L.TA;

  const int n_chunks = (a.B + NB - 1) / NB;
  const int chunk = blockIdx.x % n_chunks;
  const int rh = blockIdx.x / n_chunks;
  const int r = rh / a.H, h = rh % a.H;
  const int b0 = chunk * NB;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = a.t, n_anc = t - 1;

  if (warp == 8) {
    if (lane == 0) {
      for (int s = 0; s < 2; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);
      }
      mbar_init(done, 1);
      *abort_flag = 0;
      fence_barrier_init();
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_shi);
      prefetch_tmap(&tm_slo);
    }
    __syncwarp();
    tmem_alloc(holder, L.ncols);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;

  if (warp == 8) {
    // ---------------------------------------------------------------- producer + MMA issuer
    if (lane == 0) {
      auto stage_ptr = [&](int st) { return smem + size_t(st) * L.stage_bytes; };
      auto issue = [&](int ks, int st) {
        unsigned char* base = stage_ptr(st);
        mbar_arrive_expect_tx(&full[st], L.stage_bytes);
        tma_load_3d(base, &tm_shi, &full[st], ks * 64, 0, rh);
        tma_load_3d(base + L.a_bytes, &tm_slo, &full[st], ks * 64, 0, rh);
        tma_load_4d(base + 2 * L.a_bytes, &tm_q, &full[st], ks * 64, h, b0, r);
        tma_load_4d(base + 2 * L.a_bytes + NB * 128, &tm_k, &full[st], ks * 64, h, b0, r);
      };
      const uint32_t idesc = idesc_bf16_f32(128, 2 * NB);
      bool ok = true;
      for (int ks = 0; ks < L.NST; ++ks) issue(ks, ks);
      for (int ks = 0; ks < L.NSL; ++ks) {
        const int st = ks % L.NST;
        const uint32_t ph = uint32_t(ks / L.NST) & 1u;
        if (!mbar_wait_bounded(&full[st], ph)) { ok = false; break; }
        tc_fence_after();
        const uint32_t base = smem_u32(stage_ptr(st));
#pragma unroll
        for (int mt = 0; mt < (DV + 127) / 128; ++mt) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bdesc = sw128_kmajor_desc(base + 2 * L.a_bytes + kk * 32);
            const uint64_t ahi = sw128_kmajor_desc(base + mt * 16384 + kk * 32);
            const uint64_t alo = sw128_kmajor_desc(base + L.a_bytes + mt * 16384 + kk * 32);
            const uint32_t d = tmem + uint32_t(mt * 2 * NB);
            umma_bf16(d, ahi, bdesc, idesc, (ks | kk) != 0 ? 1u : 0u);
            umma_bf16(d, alo, bdesc, idesc, 1u);
          }
        }
        umma_commit(&empty[st]);
        if (ks + L.NST < L.NSL) {
          if (!mbar_wait_bounded(&empty[st], ph)) { ok = false; break; }
          issue(ks + L.NST, st);
        }
      }
      umma_commit(done);
      if (!ok) {
        *abort_flag = 1;
        report_error(a.err, OLA_ERR_TIMEOUT, 1, t);
      }
    }
  } else {
    // ---------------------------------------------------------------- per-beam scalars
    for (int bl = warp; bl < NB; bl += 8) {
      const int b = b0 + bl;
      if (b >= a.B) continue;
      const int p = checked_parent(a, r, b);
      int my_rec = 0;
      float my_alpha = 1.f;
      if (lane < n_anc) {
        my_rec = a.C[chain_row(a, t - 2, r, p) + lane];
        my_alpha = a.A[rec_index(a, lane, r, h, my_rec)];
      }
      float x = my_alpha;   // inclusive suffix product of the chain's alphas
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_down_sync(0xffffffffu, x, off);
        if (lane + off < 32) x *= y;
      }
      const float ep = __shfl_sync(0xffffffffu, x, 0);
      const float dec = __shfl_down_sync(0xffffffffu, x, 1);
      const size_t sidx = (size_t(r) * a.B + b) * a.H + h;
      const Vec qraw = reinterpret_cast<const Vec*>(
          static_cast<const __nv_bfloat16*>(a.q) + sidx * DK)[lane];
      const Vec kraw = reinterpret_cast<const Vec*>(
          static_cast<const __nv_bfloat16*>(a.k) + sidx * DK)[lane];
      float qv[EPL], kv[EPL];
      unpack_bf16<EPL>(qraw, qv);
      unpack_bf16<EPL>(kraw, kv);
      for (int s = 0; s < n_anc; ++s) {
        const int rs = __shfl_sync(0xffffffffu, my_rec, s);
        const Vec jraw = reinterpret_cast<const Vec*>(
            static_cast<const __nv_bfloat16*>(a.Kr) + rec_index(a, s, r, h, rs) * DK)[lane];
        float kj[EPL];
        unpack_bf16<EPL>(jraw, kj);
        float dk = 0.f, dq = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          dk = fmaf(kj[e], kv[e], dk);
          dq = fmaf(kj[e], qv[e], dq);
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
#pragma unroll
      for (int e = 0; e < EPL; ++e) c0 = fmaf(kv[e], qv[e], c0);
      c0 = warp_sum(c0);
      const float alpha = expf(a.g[sidx]);
      if (lane == 0) {
        sc[bl * 4 + 0] = ep;
        sc[bl * 4 + 1] = alpha;
        sc[bl * 4 + 2] = a.beta[sidx];
        sc[bl * 4 + 3] = c0;
        a.A[rec_index(a, t - 1, r, h, b)] = alpha;
      }
      reinterpret_cast<Vec*>(static_cast<__nv_bfloat16*>(a.Kr) +
                             rec_index(a, t - 1, r, h, b) * DK)[lane] = kraw;
      if (h == 0 && lane < t) a.C[chain_row(a, t - 1, r, b) + lane] = (lane < n_anc) ? my_rec : b;
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");   // tables complete (epilogue warps only)

    // ---------------------------------------------------------------- epilogue
    const bool have_d = mbar_wait_bounded(done, 0);
    if (!have_d) report_error(a.err, OLA_ERR_TIMEOUT, 2, t);
    tc_fence_after();
    constexpr int MT = (DV + 127) / 128;
    const int quarter = warp & 3, grp = warp >> 2;
    const int mt = (MT == 2) ? grp : 0;
    const int bl_lo = (MT == 2) ? 0 : grp * (NB / 2);
    const int bl_hi = (MT == 2) ? NB : bl_lo + NB / 2;
    const int i = mt * 128 + quarter * 32 + lane;
    if (have_d && *abort_flag == 0 && mt * 128 + quarter * 32 < DV) {
      const uint32_t tbase = tmem + (uint32_t(quarter * 32) << 16) + uint32_t(mt * 2 * NB);
      for (int bb = bl_lo; bb < bl_hi; bb += 8) {
        if (b0 + bb >= a.B) break;
        float yq[8], yk[8];
        tmem_ld8x2(tbase + bb, tbase + NB + bb, yq, yk);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int bl = bb + j, b = b0 + bl;
          if (b >= a.B) break;
          const float ep = sc[bl * 4 + 0], alpha = sc[bl * 4 + 1], beta = sc[bl * 4 + 2],
                      c0 = sc[bl * 4 + 3];
          float u = ep * yk[j];
          float qa = ep * yq[j];
          for (int s = 0; s < n_anc; ++s) {
            const float wv =
                __ldg(a.W + rec_index(a, s, r, h, rec[bl * TA + s]) * size_t(DV) + i);
            u = fmaf(cu[bl * TA + s], wv, u);
            qa = fmaf(cq[bl * TA + s], wv, qa);
          }
          const size_t sidx = (size_t(r) * a.B + b) * a.H + h;
          const float vi = __bfloat162float(static_cast<const __nv_bfloat16*>(a.v)[sidx * DV + i]);
          const float w = beta * (vi - alpha * u);
          a.o[sidx * DV + i] = fmaf(alpha, qa, c0 * w);
          a.W[rec_index(a, t - 1, r, h, b) * size_t(DV) + i] = w;
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, L.ncols);
  }
}

// ------------------------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

int tc_pick_nb(int B) { return B >= 64 ? 64 : (B >= 32 ? 32 : 16); }

// S_hi / S_lo: [R*H][MROWS][d_k] bf16, rows >= d_v zero. Box: 64 x MROWS.
bool make_state_map(CUtensorMap* map, const void* base, int RH, int d_k, int d_v) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const int mrows = ((d_v + 127) / 128) * 128;
  cuuint64_t dims[3] = {cuuint64_t(d_k), cuuint64_t(mrows), cuuint64_t(RH)};
  cuuint64_t strides[2] = {cuuint64_t(d_k) * 2, cuuint64_t(mrows) * d_k * 2};
  cuuint32_t box[3] = {64, cuuint32_t(mrows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// q or k: [R][B][H][d_k] bf16. Box: 64 x 1 x NB x 1 (one 64-wide slice of NB beams).
static bool make_input_map(CUtensorMap* map, const void* base, int R, int B, int H, int d_k,
                           int NB) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {cuuint64_t(d_k), cuuint64_t(H), cuuint64_t(B), cuuint64_t(R)};
  cuuint64_t strides[3] = {cuuint64_t(d_k) * 2, cuuint64_t(H) * d_k * 2,
                           cuuint64_t(B) * H * d_k * 2};
  cuuint32_t box[4] = {64, 1, cuuint32_t(NB), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

__global__ void split_state_kernel(const float* __restrict__ S, __nv_bfloat16* __restrict__ hi,
                                   __nv_bfloat16* __restrict__ lo, int RH, int d_k, int d_v,
                                   int mrows) {
  const size_t n = size_t(RH) * mrows * d_k;
  for (size_t idx = blockIdx.x * size_t(blockDim.x) + threadIdx.x; idx < n;
       idx += size_t(gridDim.x) * blockDim.x) {
    const int e = int(idx % d_k);
    const int i = int((idx / d_k) % mrows);
    const size_t rh = idx / (size_t(d_k) * mrows);
    float s = 0.f;
    if (i < d_v) s = S[(rh * d_v + i) * d_k + e];
    const __nv_bfloat16 sh = __float2bfloat16_rn(s);
    hi[idx] = sh;
    lo[idx] = __float2bfloat16_rn(s - __bfloat162float(sh));
  }
}

cudaError_t launch_split_state(const float* S, void* hi, void* lo, int RH, int d_k, int d_v,
                               cudaStream_t stream) {
  const int mrows = ((d_v + 127) / 128) * 128;
  split_state_kernel<<<1184, 256, 0, stream>>>(S, static_cast<__nv_bfloat16*>(hi),
                                               static_cast<__nv_bfloat16*>(lo), RH, d_k, d_v,
                                               mrows);
  return cudaGetLastError();
}

size_t replay_tc_smem(int d_k, int d_v, int B, int T_max) {
  return tc_layout(d_k, d_v, tc_pick_nb(B), T_max).bytes;
}

template <int DK, int DV>
static cudaError_t launch_tc_t(const CUtensorMap& mq, const CUtensorMap& mk,
                               const CUtensorMap& mhi, const CUtensorMap& mlo, const StepArgs& a,
                               int NB, cudaStream_t stream) {
  const TcLayout L = tc_layout(DK, DV, NB, a.T_max);
  const int n_chunks = (a.B + NB - 1) / NB;
  const unsigned grid = unsigned(a.R) * a.H * n_chunks;
  cudaFuncSetAttribute(replay_tc_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       int(L.bytes));
  replay_tc_kernel<DK, DV><<<grid, kTcThreads, L.bytes, stream>>>(mq, mk, mhi, mlo, a, NB);
  return cudaGetLastError();
}

cudaError_t launch_replay_tc(const StepArgs& a, const CUtensorMap& mhi, const CUtensorMap& mlo,
                             cudaStream_t stream) {
  const int NB = tc_pick_nb(a.B);
  CUtensorMap mq, mk;
  if (!make_input_map(&mq, a.q, a.R, a.B, a.H, a.d_k, NB) ||
      !make_input_map(&mk, a.k, a.R, a.B, a.H, a.d_k, NB))
    return cudaErrorInvalidValue;
#define OLA_TC_CASE(DK_, DV_) \
  if (a.d_k == DK_ && a.d_v == DV_) return launch_tc_t<DK_, DV_>(mq, mk, mhi, mlo, a, NB, stream);
  OLA_TC_CASE(64, 64) OLA_TC_CASE(64, 128) OLA_TC_CASE(64, 256)
  OLA_TC_CASE(128, 64) OLA_TC_CASE(128, 128) OLA_TC_CASE(128, 256)
  OLA_TC_CASE(256, 64) OLA_TC_CASE(256, 128) OLA_TC_CASE(256, 256)
#undef OLA_TC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace ola
