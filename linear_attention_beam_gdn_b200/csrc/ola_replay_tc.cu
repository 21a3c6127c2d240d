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
// Beams are visited in the depth-first order of the beam tree (see ola_plan.cu): a CTA takes
// one (request, head) and NB consecutive depth-first positions, so the beams of a CTA, and of
// neighbouring CTAs, share most of their ancestors and the gathered records stay in L1/L2.
//
// CTA roles (8 worker warps, plus a 9th control warp only for the pipelined variant):
//   phase 1  every worker lane (position j of its warp, slice g of d_k) loads its slice of
//            q_t and k_t (16-byte loads, a lane group covers a whole row), keeps it in
//            registers and writes it into the MMA's B tile in shared memory (K-major, 128-byte
//            swizzle, one tile per 64-wide K slice); the warp then signals the MMA issuer.
//   MMA      S_hi and S_lo K slices arrive by TMA (issued at CTA start); one thread issues
//            M = 128, N = 2 NB, K = 16 tcgen05.mma, hi and lo into one fp32 accumulator per
//            M tile. Resident variant (d_k, d_v <= 128): every slice stays in shared memory
//            and worker warp 0 issues the MMAs right after phase 1. Pipelined variant: a
//            control warp streams the slices through a two-stage ring.
//   phase 2  chain gather (record rows and alphas of every (position, ancestor) pair), the
//            alpha suffix products, and the dot products k_j . k_t, k_j . q_t computed by
//            the lane group that holds k_t, q_t (16-byte loads of k_j, fp32 FMA, a shuffle
//            tree over the group); appends k_t, alpha_t and the chain row.
//   phase 3  thread = row i of d_v (tensor-memory lane): for groups of 8 positions, the
//            ancestors' w_j rows and v are loaded together (no predication: positions past
//            B point at row 0), then u, w_t, o_t and coalesced stores of o and w_t.
// Every wait is bounded; on timeout the kernel records OLA_ERR_TIMEOUT and finishes.
#include "ola_device.cuh"

namespace ola {

// per-position scalars (32 bytes)
struct PosRec {
  int b;         // beam index, -1 past the end of the step
  int io;        // row of v and o: (r B + b) H + h (0 past the end)
  int wnew;      // record row of the new w_t: ((t-1) R + r) H + h) B + b
  int p;         // parent beam
  float ep;      // product of every alpha on the chain
  float alpha, beta, c0;   // alpha_t, beta_t, k_t . q_t
};

// one (position, ancestor) entry (16 bytes)
struct AncRec {
  int row;       // record row of the ancestor
  float cu;      // (prod_{i>j} alpha_i) (k_j . k_t)   [alpha_j before phase 2's dots]
  float cq;      // (prod_{i>j} alpha_i) (k_j . q_t)   [decay product before the dots]
  int rec;       // beam index of the ancestor record
};

struct TcLayout {
  int MT, MROWS, NSL, NST, NB, TA;
  uint32_t a_bytes, stage_bytes, x_slice_bytes, ncols;
  size_t x_off, bar_off, ps_off, tab_off, bytes;
};

__host__ __device__ constexpr bool tc_resident(int d_k, int d_v) { return d_k <= 128 && d_v <= 128; }

__host__ __device__ inline int tc_pick_nb(int B, int d_k) {
  return (d_k >= 256 || B < 64) ? 32 : 64;
}

__host__ __device__ inline TcLayout tc_layout(int d_k, int d_v, int NB, int T_max) {
  TcLayout L;
  L.MT = (d_v + 127) / 128;
  L.MROWS = L.MT * 128;
  L.NSL = d_k / 64;
  L.NST = tc_resident(d_k, d_v) ? L.NSL : (L.NSL < 2 ? L.NSL : 2);
  L.NB = NB;
  L.TA = T_max > 1 ? T_max - 1 : 1;
  L.a_bytes = uint32_t(L.MROWS) * 128u;
  L.stage_bytes = 2u * L.a_bytes;                       // S_hi and S_lo slices
  L.x_slice_bytes = uint32_t(2 * NB) * 128u;            // [q; k] rows of one K slice
  uint32_t need = uint32_t(L.MT * 2 * NB), c = 32;
  while (c < need) c <<= 1;
  L.ncols = c;
  L.x_off = size_t(L.NST) * L.stage_bytes;
  L.bar_off = L.x_off + size_t(L.NSL) * L.x_slice_bytes;
  L.ps_off = L.bar_off + 128;                           // 16 x 8-byte barrier / flag slots
  L.tab_off = L.ps_off + sizeof(PosRec) * NB;
  L.bytes = L.tab_off + sizeof(AncRec) * NB * L.TA + 1024;  // + slack for 1024-B alignment
  return L;
}

__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

template <int DK, int DV, int NB, bool CTRL>
__global__ void __launch_bounds__(CTRL ? 288 : 256, CTRL ? 1 : 2)
replay_tc_kernel(const __grid_constant__ CUtensorMap tm_shi,
                 const __grid_constant__ CUtensorMap tm_slo, StepArgs a) {
  constexpr int MT = (DV + 127) / 128;
  constexpr int NSL = DK / 64;
  constexpr int PW = NB / 8;          // positions per worker warp
  constexpr int LPP = 32 / PW;        // lanes per position
  constexpr int DPL = DK / LPP;       // d_k elements per lane
  constexpr int CPL = DPL / 8;        // 16-byte chunks per lane
  static_assert(CPL >= 1 && CPL * 8 == DPL, "lane slice must be whole 16-byte chunks");
  static_assert(CTRL || tc_resident(DK, DV), "resident variant needs d_k, d_v <= 128");

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align_smem_1024(smem_raw);
  const TcLayout L = tc_layout(DK, DV, NB, a.T_max);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);   // [4]
  uint64_t* empty = full + 4;                                        // [2]
  uint64_t* xfull = full + 6;
  uint64_t* done = full + 7;
  uint32_t* holder = reinterpret_cast<uint32_t*>(full + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + 9);
  unsigned char* xs = smem + L.x_off;
  PosRec* ps = reinterpret_cast<PosRec*>(smem + L.ps_off);          // [NB]
  AncRec* tab = reinterpret_cast<AncRec*>(smem + L.tab_off);        // [NB][TA]
  const int TA = L.TA;

  const int n_chunks = (a.B + NB - 1) / NB;
  const int chunk = blockIdx.x % n_chunks;
  const int rh = blockIdx.x / n_chunks;
  const int r = rh / a.H, h = rh % a.H;
  const int c0 = chunk * NB;                      // first depth-first position of the CTA
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = a.t, n_anc = t - 1;
  const int ctl_warp = CTRL ? 8 : 0;

  auto issue_slice = [&](int ks, int st) {
    unsigned char* base = smem + size_t(st) * L.stage_bytes;
    mbar_arrive_expect_tx(&full[st], L.stage_bytes);
    tma_load_3d(base, &tm_shi, &full[st], ks * 64, 0, rh);
    tma_load_3d(base + L.a_bytes, &tm_slo, &full[st], ks * 64, 0, rh);
  };
  auto issue_mmas = [&](int ks, int st) {
    const uint32_t idesc = idesc_bf16_f32(128, 2 * NB);
    const uint32_t abase = smem_u32(smem + size_t(st) * L.stage_bytes);
    const uint32_t xbase = smem_u32(xs + size_t(ks) * L.x_slice_bytes);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t bdesc = sw128_kmajor_desc(xbase + kk * 32);
        const uint64_t ahi = sw128_kmajor_desc(abase + mt * 16384 + kk * 32);
        const uint64_t alo = sw128_kmajor_desc(abase + L.a_bytes + mt * 16384 + kk * 32);
        const uint32_t d = *holder + uint32_t(mt * 2 * NB);
        umma_bf16(d, ahi, bdesc, idesc, (ks | kk) != 0 ? 1u : 0u);
        umma_bf16(d, alo, bdesc, idesc, 1u);
      }
    }
  };

  if (warp == ctl_warp) {
    if (lane == 0) {
      for (int s = 0; s < 4; ++s) mbar_init(&full[s], 1);
      for (int s = 0; s < 2; ++s) mbar_init(&empty[s], 1);
      mbar_init(xfull, 8);
      mbar_init(done, 1);
      *abort_flag = 0;
      fence_barrier_init();
      prefetch_tmap(&tm_shi);
      prefetch_tmap(&tm_slo);
      for (int ks = 0; ks < L.NST; ++ks) issue_slice(ks, ks);
    }
    __syncwarp();
    tmem_alloc(holder, L.ncols);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;

  if (CTRL && warp == 8) {
    // ---------------------------------------------------------------- pipelined MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait_bounded(xfull, 0);
      for (int ks = 0; ok && ks < NSL; ++ks) {
        const int st = ks % L.NST;
        const uint32_t ph = uint32_t(ks / L.NST) & 1u;
        if (!mbar_wait_bounded(&full[st], ph)) { ok = false; break; }
        tc_fence_after();
        issue_mmas(ks, st);
        umma_commit(&empty[st]);
        if (ks + L.NST < NSL) {
          if (!mbar_wait_bounded(&empty[st], ph)) { ok = false; break; }
          issue_slice(ks + L.NST, st);
        }
      }
      umma_commit(done);
      if (!ok) {
        *abort_flag = 1;
        report_error(a.err, OLA_ERR_TIMEOUT, 1, t);
      }
    }
  } else {
    // ---------------------------------------------------------------- phase 1: q, k
    const int j = lane / LPP, g = lane % LPP;
    const int pl = warp * PW + j;                 // this lane's position in the chunk
    const int pos = c0 + pl;
    const bool valid = pos < a.B;
    int b = 0, p = 0;
    if (valid) {
      b = a.perm[size_t(r) * a.B + pos];
      p = a.pparent[size_t(r) * a.B + pos];
    }
    const int io = valid ? (r * a.B + b) * a.H + h : 0;
    uint4 qv[CPL], kv[CPL];
    {
      const uint4* qrow = reinterpret_cast<const uint4*>(
          static_cast<const __nv_bfloat16*>(a.q) + size_t(io) * DK + g * DPL);
      const uint4* krow = reinterpret_cast<const uint4*>(
          static_cast<const __nv_bfloat16*>(a.k) + size_t(io) * DK + g * DPL);
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        qv[c] = valid ? qrow[c] : make_uint4(0u, 0u, 0u, 0u);
        kv[c] = valid ? krow[c] : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const int e = g * DPL + 8 * c;
        const int ks = e / 64, ch = (e % 64) / 8;
        unsigned char* sl = xs + size_t(ks) * L.x_slice_bytes;
        const int nq = pl, nk = NB + pl;
        *reinterpret_cast<uint4*>(sl + nq * 128 + ((ch ^ (nq & 7)) * 16)) = qv[c];
        *reinterpret_cast<uint4*>(sl + nk * 128 + ((ch ^ (nk & 7)) * 16)) = kv[c];
      }
    }
    if (g == 0) {
      PosRec pr;
      pr.b = valid ? b : -1;
      pr.io = io;
      pr.wnew = valid ? int(rec_index(a, t - 1, r, h, b)) : 0;
      pr.p = p;
      pr.ep = 1.f;
      pr.alpha = 0.f;
      pr.beta = 0.f;
      pr.c0 = 0.f;
      ps[pl] = pr;
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(xfull);
    if (!CTRL && warp == 0) {
      if (lane == 0) {
        bool ok = mbar_wait_bounded(xfull, 0);
        for (int ks = 0; ok && ks < NSL; ++ks) {
          if (!mbar_wait_bounded(&full[ks], 0)) { ok = false; break; }
          tc_fence_after();
          issue_mmas(ks, ks);
        }
        umma_commit(done);
        if (!ok) {
          *abort_flag = 1;
          report_error(a.err, OLA_ERR_TIMEOUT, 1, t);
        }
      }
      __syncwarp();
    }

    // ---------------------------------------------------------------- phase 2: chains, dots
    for (int idx = lane; idx < PW * n_anc; idx += 32) {
      const int jj = idx / n_anc, s = idx % n_anc;
      const int pl2 = warp * PW + jj;
      const PosRec& pr = ps[pl2];
      int rs = 0;
      float al = 1.f;
      if (pr.b >= 0) {
        rs = a.C[chain_row(a, t - 2, r, pr.p) + s];
        al = a.A[rec_index(a, s, r, h, rs)];
      }
      AncRec e;
      e.row = int(rec_index(a, s, r, h, rs));
      e.cu = al;
      e.cq = 0.f;
      e.rec = rs;
      tab[pl2 * TA + s] = e;
    }
    __syncwarp();
    float ep = 1.f;
    if (g == 0) {                                  // decay products along the chain
      float x = 1.f;
      for (int s = n_anc - 1; s >= 0; --s) {
        tab[pl * TA + s].cq = x;                   // prod_{i>s} alpha_i
        x *= tab[pl * TA + s].cu;
      }
      ep = x;
    }
    __syncwarp();
    const __nv_bfloat16* krec = static_cast<const __nv_bfloat16*>(a.Kr);
#pragma unroll 2
    for (int s = 0; s < n_anc; ++s) {
      const int row = tab[pl * TA + s].row;
      const uint4* kj = reinterpret_cast<const uint4*>(krec + size_t(row) * DK + g * DPL);
      float dk = 0.f, dq = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const uint4 x = kj[c];
        const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
        const uint32_t kw[4] = {kv[c].x, kv[c].y, kv[c].z, kv[c].w};
        const uint32_t qw[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          dk = fmaf(bf_lo(xw[m]), bf_lo(kw[m]), dk);
          dk = fmaf(bf_hi(xw[m]), bf_hi(kw[m]), dk);
          dq = fmaf(bf_lo(xw[m]), bf_lo(qw[m]), dq);
          dq = fmaf(bf_hi(xw[m]), bf_hi(qw[m]), dq);
        }
      }
#pragma unroll
      for (int off = LPP / 2; off > 0; off >>= 1) {
        dk += __shfl_xor_sync(0xffffffffu, dk, off);
        dq += __shfl_xor_sync(0xffffffffu, dq, off);
      }
      if (g == 0) {
        const float dec = tab[pl * TA + s].cq;
        tab[pl * TA + s].cu = dec * dk;
        tab[pl * TA + s].cq = dec * dq;
      }
    }
    float c0d = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const uint32_t kw[4] = {kv[c].x, kv[c].y, kv[c].z, kv[c].w};
      const uint32_t qw[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        c0d = fmaf(bf_lo(kw[m]), bf_lo(qw[m]), c0d);
        c0d = fmaf(bf_hi(kw[m]), bf_hi(qw[m]), c0d);
      }
    }
#pragma unroll
    for (int off = LPP / 2; off > 0; off >>= 1) c0d += __shfl_xor_sync(0xffffffffu, c0d, off);
    if (valid) {
      const size_t sidx = size_t(io);
      if (g == 0) {
        const float alpha = expf(a.g[sidx]);
        ps[pl].ep = ep;
        ps[pl].alpha = alpha;
        ps[pl].beta = a.beta[sidx];
        ps[pl].c0 = c0d;
        a.A[rec_index(a, t - 1, r, h, b)] = alpha;
      }
      uint4* kdst = reinterpret_cast<uint4*>(const_cast<__nv_bfloat16*>(krec) +
                                             rec_index(a, t - 1, r, h, b) * DK + g * DPL);
#pragma unroll
      for (int c = 0; c < CPL; ++c) kdst[c] = kv[c];
      if (h == 0)
        for (int s = g; s < t; s += LPP)
          a.C[chain_row(a, t - 1, r, b) + s] = (s < n_anc) ? tab[pl * TA + s].rec : b;
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");   // tables complete (worker warps only)

    // ---------------------------------------------------------------- phase 3: epilogue
    const bool have_d = mbar_wait_bounded(done, 0);
    if (!have_d) report_error(a.err, OLA_ERR_TIMEOUT, 2, t);
    tc_fence_after();
    const int quarter = warp & 3, grp = warp >> 2;
    const int mt = (MT == 2) ? grp : 0;
    const int bl_lo = (MT == 2) ? 0 : grp * (NB / 2);
    const int bl_hi = (MT == 2) ? NB : bl_lo + NB / 2;
    const int i = mt * 128 + quarter * 32 + lane;
    if (have_d && *abort_flag == 0 && mt * 128 + quarter * 32 < DV) {
      const uint32_t tbase = tmem + (uint32_t(quarter * 32) << 16) + uint32_t(mt * 2 * NB);
      const __nv_bfloat16* vg = static_cast<const __nv_bfloat16*>(a.v);
      const float* Wg = a.W;
      for (int bb = bl_lo; bb < bl_hi; bb += 8) {
        if (c0 + bb >= a.B) break;
        float yq[8], yk[8];
        tmem_ld8x2(tbase + bb, tbase + NB + bb, yq, yk);
        float u[8], qa[8], vv[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const float e = ps[bb + jj].ep;
          u[jj] = e * yk[jj];
          qa[jj] = e * yq[jj];
          vv[jj] = __bfloat162float(vg[size_t(ps[bb + jj].io) * DV + i]);
        }
#pragma unroll 2
        for (int s = 0; s < n_anc; ++s) {
          float wv[8];
          float2 cf[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const AncRec e = tab[(bb + jj) * TA + s];
            cf[jj] = make_float2(e.cu, e.cq);
            wv[jj] = __ldg(Wg + size_t(e.row) * DV + i);
          }
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            u[jj] = fmaf(cf[jj].x, wv[jj], u[jj]);
            qa[jj] = fmaf(cf[jj].y, wv[jj], qa[jj]);
          }
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const PosRec pr = ps[bb + jj];
          if (pr.b >= 0) {
            const float w = pr.beta * (vv[jj] - pr.alpha * u[jj]);
            a.o[size_t(pr.io) * DV + i] = fmaf(pr.alpha, qa[jj], pr.c0 * w);
            a.W[size_t(pr.wnew) * DV + i] = w;
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == ctl_warp) {
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

// Rows of a 2-D bf16 matrix [rows][cols] (row stride row_bytes) for row gathers: box of 64
// columns x 1 row, 128-byte swizzle (tile::gather4 loads four rows per instruction).
bool make_rows_map(CUtensorMap* map, const void* base, uint64_t rows, int cols,
                   uint64_t row_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(row_bytes)};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t es[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
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
  return tc_layout(d_k, d_v, tc_pick_nb(B, d_k), T_max).bytes;
}

template <int DK, int DV, int NB>
static cudaError_t launch_tc_t(const CUtensorMap& mhi, const CUtensorMap& mlo, const StepArgs& a,
                               cudaStream_t stream) {
  constexpr bool CTRL = !tc_resident(DK, DV);
  const TcLayout L = tc_layout(DK, DV, NB, a.T_max);
  const int n_chunks = (a.B + NB - 1) / NB;
  const unsigned grid = unsigned(a.R) * a.H * n_chunks;
  auto kern = replay_tc_kernel<DK, DV, NB, CTRL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(L.bytes));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  kern<<<grid, CTRL ? 288 : 256, L.bytes, stream>>>(mhi, mlo, a);
  return cudaGetLastError();
}

cudaError_t launch_plan(const StepArgs& a, cudaStream_t stream);

cudaError_t launch_replay_tc(const StepArgs& a, const CUtensorMap& mhi, const CUtensorMap& mlo,
                             cudaStream_t stream) {
  const int NB = tc_pick_nb(a.B, a.d_k);
  cudaError_t e = launch_plan(a, stream);
  if (e != cudaSuccess) return e;
#define OLA_TC_CASE(DK_, DV_, NB_)                                   \
  if (a.d_k == DK_ && a.d_v == DV_ && NB == NB_)                     \
    return launch_tc_t<DK_, DV_, NB_>(mhi, mlo, a, stream);
  OLA_TC_CASE(64, 64, 32) OLA_TC_CASE(64, 128, 32) OLA_TC_CASE(64, 256, 32)
  OLA_TC_CASE(128, 64, 32) OLA_TC_CASE(128, 128, 32) OLA_TC_CASE(128, 256, 32)
  OLA_TC_CASE(256, 64, 32) OLA_TC_CASE(256, 128, 32) OLA_TC_CASE(256, 256, 32)
  OLA_TC_CASE(64, 64, 64) OLA_TC_CASE(64, 128, 64) OLA_TC_CASE(64, 256, 64)
  OLA_TC_CASE(128, 64, 64) OLA_TC_CASE(128, 128, 64) OLA_TC_CASE(128, 256, 64)
#undef OLA_TC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace ola
