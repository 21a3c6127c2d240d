// Projection-replay decode step on the tcgen05 tensor cores, beam-major (sm_100a;
// d_k, d_v <= 128).
//
// Mathematics as in ola_replay_simt.cu ("Scientific Impact Assessment: OneLA", §1 Core
// Contribution: one shared post-prefill state, append-only transition records, projection
// replay through the key and query contractions, one fused kernel reusing the shared state
// across beams). For beam b with parent chain j = 1..t-1:
//     Y_q = S_ctx q_t, Y_k = S_ctx k_t                               (tensor cores)
//     u   = e Y_k + sum_j d_j (k_j . k_t) w_j,   w_t = beta (v_t - alpha u)
//     o_t = alpha (e Y_q + sum_j d_j (k_j . q_t) w_j) + (k_t . q_t) w_t
// with d_j = prod_{i>j} alpha_i and e = prod_j alpha_j.
//
// Contraction: D[beam][i] = sum_k X[beam][k] S[i][k], M = the CTA's 64 (or 128) beams (A =
// their q, then k, rows), N = d_v (B = S_ctx), K = d_k, both operands K-major with the
// 128-byte swizzle. S_ctx is split once into bf16 hi + lo: two MMAs into one fp32 accumulator
// (|error| ~ 2^-17 |S|). D_q, D_k live in tensor memory, one beam per lane, d_v columns. With
// 64 beams a CTA needs ~107 KB of shared memory and 256 threads, so two CTAs share an SM and
// one's loads overlap the other's stores.
//
// Everything else is warp-per-beam: a warp owns 8 consecutive depth-first positions of the
// CTA (ola_plan.cu) through all phases, and lane l owns elements [l E, (l+1) E) of every d_k or
// d_v row of those beams. Every record / input / output row is then one coalesced warp access,
// and every per-beam quantity (parent, chain, decay products, dot products) is warp-uniform:
//   phase 1  q_t, k_t rows -> registers and the swizzled A tiles; k_t, alpha_t and the chain
//            row appended; the parent's chain (record rows, alphas) into a per-beam table;
//            k_t . q_t.
//   MMA      warp 0 lane 0, once the S_ctx slices (TMA at CTA start) and the A tiles are in.
//   phase 2  k_j . k_t and k_j . q_t for every ancestor on warp-level tensor-core MMA
//            (16 (beam, ancestor) rows x 8 beams per m16n8k16), then the decay pass.
//   D        tensor memory -> shared memory transposed to beam-major rows, reusing the space
//            of the S and A tiles (XOR-swizzled by row: conflict-free both ways).
//   phase 3  per beam: Y rows, ancestors' w_j rows, v row -> u, w_t, o_t -> o and w_t rows.
// Every wait is bounded; on timeout the kernel records OLA_ERR_TIMEOUT and finishes.
#include "ola_device.cuh"

namespace ola {

constexpr int kPosPPW = 8;             // positions per warp

struct AncPos {          // one (position, ancestor) entry, 16 bytes
  int row;               // record row of the ancestor
  float alpha;           // its alpha
  float cu, cq;          // d_j (k_j . k_t), d_j (k_j . q_t)   (raw dots before the decay pass)
};

struct PosScal {         // per-position scalars, 32 bytes
  int b, io, wnew, pad;
  float ep, alpha, beta, c0;
};

struct PosLayout {
  int NSL, TA;
  uint32_t s_bytes, x_bytes, ncols;   // one hi (or lo) slice of S; one q (or k) slice of X
  size_t x_off, y_bytes, bar_off, ps_off, tab_off, bytes;
};

__host__ __device__ inline PosLayout pos_layout(int d_k, int d_v, int T_max, int NB) {
  PosLayout L;
  L.NSL = d_k / 64;
  L.TA = T_max > 1 ? T_max - 1 : 1;
  L.s_bytes = 128u * 128u;                       // S rows padded to 128 (zero rows past d_v)
  L.x_bytes = uint32_t(NB) * 128u;
  uint32_t c = 32;
  while (c < uint32_t(2 * d_v)) c <<= 1;
  L.ncols = c;
  L.x_off = size_t(L.NSL) * 2 * L.s_bytes;
  const size_t sx = L.x_off + size_t(L.NSL) * 2 * L.x_bytes;
  L.y_bytes = size_t(NB) * d_v * 4;
  L.bar_off = sx > 2 * L.y_bytes ? sx : 2 * L.y_bytes;
  L.ps_off = L.bar_off + 64;
  L.tab_off = L.ps_off + sizeof(PosScal) * NB;
  L.bytes = L.tab_off + sizeof(AncPos) * NB * L.TA + 1024;
  return L;
}

template <int N> struct Words;                  // N 32-bit words moved as one access
template <> struct Words<1> { using T = uint32_t; };
template <> struct Words<2> { using T = uint2; };
template <> struct Words<4> { using T = uint4; };

template <int N>
__device__ __forceinline__ void unpack_words(const typename Words<N>::T& v, uint32_t (&w)[N]) {
  const uint32_t* p = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
  for (int i = 0; i < N; ++i) w[i] = p[i];
}

__device__ __forceinline__ float bfl(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bfh(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// sum over the lane's bf16 pairs of a . b
template <int N>
__device__ __forceinline__ float dot_bf16(const typename Words<N>::T& x,
                                          const typename Words<N>::T& y, float acc) {
  uint32_t a[N], b[N];
  unpack_words<N>(x, a);
  unpack_words<N>(y, b);
#pragma unroll
  for (int i = 0; i < N; ++i) {
    acc = fmaf(bfl(a[i]), bfl(b[i]), acc);
    acc = fmaf(bfh(a[i]), bfh(b[i]), acc);
  }
  return acc;
}

// NB = beams per CTA = MMA M: 128 (16 warps, one CTA per SM) or 64 (8 warps, two per SM).
template <int DK, int DV, int NB>
__global__ void __launch_bounds__(NB * 4, NB == 64 ? 2 : 1)
replay_pos_kernel(const __grid_constant__ CUtensorMap tm_shi,
                  const __grid_constant__ CUtensorMap tm_slo, StepArgs a) {
  constexpr int NSL = DK / 64;
  constexpr int EPL = DK / 32;         // d_k elements (bf16) per lane: 2 or 4
  constexpr int KW = EPL / 2;          // 32-bit words per lane of a d_k row
  constexpr int VPL = DV / 32;         // d_v values per lane: 2 or 4
  constexpr int R4 = DV / 4;           // tensor-memory columns per thread in the transpose
  constexpr int PPW = kPosPPW;
  constexpr int YCH = DV / 4;          // 16-byte chunks per transposed row
  using KVec = typename Words<KW>::T;       // a lane's slice of a bf16 d_k row
  using FVec = typename Words<VPL>::T;      // a lane's slice of an fp32 d_v row
  using VVec = typename Words<VPL / 2>::T;  // a lane's slice of a bf16 d_v row
  static_assert(DK <= 128 && DV <= 128 && EPL >= 2 && VPL >= 2, "geometry");

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align_smem_1024(smem_raw);
  const PosLayout L = pos_layout(DK, DV, a.T_max, NB);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);   // [2]
  uint64_t* done = full + 2;
  uint32_t* holder = reinterpret_cast<uint32_t*>(full + 3);
  PosScal* ps = reinterpret_cast<PosScal*>(smem + L.ps_off);        // [NB]
  AncPos* tab = reinterpret_cast<AncPos*>(smem + L.tab_off);        // [NB][TA]
  const int TA = L.TA;

  const int n_chunks = (a.B + NB - 1) / NB;
  const int chunk = blockIdx.x % n_chunks;
  const int rh = blockIdx.x / n_chunks;
  const int r = rh / a.H, h = rh % a.H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c0 = chunk * NB;
  const int t = a.t, n_anc = t - 1;
  const int p0 = warp * PPW;                       // this warp's first position

  auto s_tile = [&](int ks, int lo) { return smem + size_t(ks) * 2 * L.s_bytes + lo * L.s_bytes; };
  auto x_tile = [&](int ks, int kside) {
    return smem + L.x_off + size_t(ks) * 2 * L.x_bytes + kside * L.x_bytes;
  };
  // transposed accumulator row p of side 0 (Y_q) or 1 (Y_k): byte address of 16-byte chunk ch
  auto ychunk = [&](int side, int p, int ch) {
    return smem + size_t(side) * L.y_bytes + size_t(p) * DV * 4 +
           size_t((ch ^ (p & (YCH - 1))) * 16);
  };

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < 2; ++s) mbar_init(&full[s], 1);
      mbar_init(done, 1);
      fence_barrier_init();
      prefetch_tmap(&tm_shi);
      prefetch_tmap(&tm_slo);
      for (int ks = 0; ks < NSL; ++ks) {
        mbar_arrive_expect_tx(&full[ks], 2 * L.s_bytes);
        tma_load_3d(s_tile(ks, 0), &tm_shi, &full[ks], ks * 64, 0, rh);
        tma_load_3d(s_tile(ks, 1), &tm_slo, &full[ks], ks * 64, 0, rh);
      }
    }
    __syncwarp();
    tmem_alloc(holder, L.ncols);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;

  // -------------------------------------------------------------------- phase 1
  // Phase 1: the beams of this warp's positions and their parents' chains (both indexed by
  // position). Phase 2: q_t, k_t rows, g, beta, the chain's alphas.
  int recs[PPW];
#pragma unroll
  for (int jj = 0; jj < PPW; ++jj) {
    const bool vj = c0 + p0 + jj < a.B;
    recs[jj] = (vj && lane < n_anc)
                   ? a.pchain[(size_t(r) * a.B + c0 + p0 + jj) * a.T_max + lane]
                   : 0;
  }
  int my_b = 0, my_io = 0;
  bool my_valid = false;
  if (lane < PPW) {                                // lane j: this warp's position j
    const int pos = c0 + p0 + lane;
    my_valid = pos < a.B;
    if (my_valid) {
      my_b = a.perm[size_t(r) * a.B + pos];
      my_io = (r * a.B + my_b) * a.H + h;
    }
  }
  int rows[PPW];
  float al[PPW];
  // record row of (step lane+1, request r, head h, beam 0): rows are this base + beam index
  const int row_base = int(rec_index(a, lane < n_anc ? lane : 0, r, h, 0));
#pragma unroll
  for (int jj = 0; jj < PPW; ++jj) {
    const bool vj = c0 + p0 + jj < a.B;
    rows[jj] = row_base + recs[jj];
    al[jj] = (vj && lane < n_anc) ? a.A[rows[jj]] : 1.f;
  }
  float my_alpha = 0.f, my_beta = 0.f;
  if (lane < PPW && my_valid) {
    my_alpha = expf(a.g[my_io]);
    my_beta = a.beta[my_io];
  }
  KVec qv[PPW], kv[PPW];
#pragma unroll
  for (int jj = 0; jj < PPW; ++jj) {
    const int io = __shfl_sync(0xffffffffu, my_io, jj);
    const bool vj = c0 + p0 + jj < a.B;
    const KVec z = {};
    qv[jj] = vj ? reinterpret_cast<const KVec*>(static_cast<const __nv_bfloat16*>(a.q) +
                                                size_t(io) * DK)[lane]
                : z;
    kv[jj] = vj ? reinterpret_cast<const KVec*>(static_cast<const __nv_bfloat16*>(a.k) +
                                                size_t(io) * DK)[lane]
                : z;
  }
#pragma unroll
  for (int jj = 0; jj < PPW; ++jj) {
    const int pn = p0 + jj;
    // A tiles: this lane's EPL elements of row pn (K slice, 16-byte chunk, byte offset)
    const int e0 = EPL * lane;
    const int ks = e0 / 64, ch = (e0 % 64) / 8, sub = (e0 % 8) * 2;
    *reinterpret_cast<KVec*>(x_tile(ks, 0) + pn * 128 + ((ch ^ (pn & 7)) * 16) + sub) = qv[jj];
    *reinterpret_cast<KVec*>(x_tile(ks, 1) + pn * 128 + ((ch ^ (pn & 7)) * 16) + sub) = kv[jj];
  }
  // chain table: record rows and alphas (lane s < n_anc); appends; k_t . q_t
  {
#pragma unroll
    for (int jj = 0; jj < PPW; ++jj) {
      const int pn = p0 + jj;
      const int bj = __shfl_sync(0xffffffffu, my_b, jj);
      const int ioj = __shfl_sync(0xffffffffu, my_io, jj);
      const bool vj = __shfl_sync(0xffffffffu, my_valid ? 1 : 0, jj) != 0;
      if (lane < n_anc) {
        tab[pn * TA + lane].row = rows[jj];
        tab[pn * TA + lane].alpha = al[jj];
      }
      float c0d = dot_bf16<KW>(kv[jj], qv[jj], 0.f);
      c0d = warp_sum(c0d);
      if (vj) {
        const size_t rnew = rec_index(a, t - 1, r, h, bj);
        reinterpret_cast<KVec*>(static_cast<__nv_bfloat16*>(a.Kr) + rnew * DK)[lane] = kv[jj];
        if (h == 0 && lane < t)
          a.C[chain_row(a, t - 1, r, bj) + lane] = (lane < n_anc) ? recs[jj] : bj;
      }
      if (lane == 0) {
        PosScal sc;
        sc.b = vj ? bj : -1;
        sc.io = ioj;
        sc.wnew = vj ? int(rec_index(a, t - 1, r, h, bj)) : 0;
        sc.pad = 0;
        sc.ep = 1.f;
        sc.alpha = 0.f;
        sc.beta = 0.f;
        sc.c0 = c0d;
        ps[pn] = sc;
      }
    }
  }
  // (every shuffle above runs on all 32 lanes, outside lane-dependent branches)
  fence_proxy_async_smem();
  __syncthreads();
  if (lane < PPW && my_valid) {
    ps[p0 + lane].alpha = my_alpha;
    ps[p0 + lane].beta = my_beta;
    a.A[rec_index(a, t - 1, r, h, my_b)] = my_alpha;
  }

  // -------------------------------------------------------------------- MMA
  if (warp == 0 && lane == 0) {
    bool ok = true;
    const uint32_t idesc = idesc_bf16_f32(NB, DV);
    for (int ks = 0; ok && ks < NSL; ++ks) {
      if (!mbar_wait_bounded(&full[ks], 0)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t aq = sw128_kmajor_desc(smem_u32(x_tile(ks, 0)) + kk * 32);
        const uint64_t ak = sw128_kmajor_desc(smem_u32(x_tile(ks, 1)) + kk * 32);
        const uint64_t bh = sw128_kmajor_desc(smem_u32(s_tile(ks, 0)) + kk * 32);
        const uint64_t bl = sw128_kmajor_desc(smem_u32(s_tile(ks, 1)) + kk * 32);
        const uint32_t acc = (ks | kk) != 0 ? 1u : 0u;
        umma_bf16(tmem, aq, bh, idesc, acc);
        umma_bf16(tmem, aq, bl, idesc, 1u);
        umma_bf16(tmem + DV, ak, bh, idesc, acc);
        umma_bf16(tmem + DV, ak, bl, idesc, 1u);
      }
    }
    umma_commit(done);
    if (!ok) report_error(a.err, OLA_ERR_TIMEOUT, 1, t);
  }

  // -------------------------------------------------------------------- phase 2: dots
  // Warp-level tensor-core MMA (m16n8k16, bf16 in, fp32 accumulate): the 16 rows of A are the
  // keys of ancestors s0 (rows 0-7) and s0+1 (rows 8-15) of the warp's 8 positions, the 8
  // columns of B are those positions' k_t (then q_t). Only the diagonal D[j][j], D[8+j][j] is
  // used. The k index is permuted consistently in A and B (the dot product is a sum) so that
  // lane (g, c) of each fragment reads whole 16-byte chunks: chunk m of a row = elements
  // [32 m + 8 c, +8), which feed virtual k-steps 2m and 2m+1.
  {
    const int gq = lane >> 2, cq4 = lane & 3;
    const int pn = p0 + gq;
    uint4 xk[DK / 32], xq[DK / 32];
#pragma unroll
    for (int m = 0; m < DK / 32; ++m) {
      const int e = 32 * m + 8 * cq4;
      const int ks = e / 64, ch = (e % 64) / 8;
      xk[m] = *reinterpret_cast<const uint4*>(x_tile(ks, 1) + pn * 128 + ((ch ^ (pn & 7)) * 16));
      xq[m] = *reinterpret_cast<const uint4*>(x_tile(ks, 0) + pn * 128 + ((ch ^ (pn & 7)) * 16));
    }
    const __nv_bfloat16* krec = static_cast<const __nv_bfloat16*>(a.Kr);
    constexpr int NP = 2;                          // ancestor pairs per round (4 rows in flight)
    for (int s0 = 0; s0 < n_anc; s0 += 2 * NP) {
      uint4 kr[2 * NP][DK / 32];
#pragma unroll
      for (int i = 0; i < 2 * NP; ++i) {
        const int s = s0 + i < n_anc ? s0 + i : s0;
        const uint4* src =
            reinterpret_cast<const uint4*>(krec + size_t(tab[pn * TA + s].row) * DK + 8 * cq4);
#pragma unroll
        for (int m = 0; m < DK / 32; ++m) kr[i][m] = src[4 * m];
      }
#pragma unroll
      for (int pr = 0; pr < NP; ++pr) {
        const uint4* ka = kr[2 * pr];
        const uint4* kb = kr[2 * pr + 1];
        float dk[4] = {0.f, 0.f, 0.f, 0.f}, dq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int m = 0; m < DK / 32; ++m) {
          mma_16816_bf16(dk, ka[m].x, kb[m].x, ka[m].y, kb[m].y, xk[m].x, xk[m].y);
          mma_16816_bf16(dq, ka[m].x, kb[m].x, ka[m].y, kb[m].y, xq[m].x, xq[m].y);
          mma_16816_bf16(dk, ka[m].z, kb[m].z, ka[m].w, kb[m].w, xk[m].z, xk[m].w);
          mma_16816_bf16(dq, ka[m].z, kb[m].z, ka[m].w, kb[m].w, xq[m].z, xq[m].w);
        }
        const int s = s0 + 2 * pr;
        if (cq4 == (gq >> 1)) {                      // this lane holds column gq = position gq
          const int o = gq & 1;
          if (s < n_anc) {
            tab[pn * TA + s].cu = dk[o];
            tab[pn * TA + s].cq = dq[o];
          }
          if (s + 1 < n_anc) {
            tab[pn * TA + s + 1].cu = dk[2 + o];
            tab[pn * TA + s + 1].cq = dq[2 + o];
          }
        }
      }
    }
  }
  __syncwarp();
  if (lane < PPW) {                  // decay products, newest ancestor first (lane = position)
    const int pn = p0 + lane;
    float x = 1.f;
    for (int s = n_anc - 1; s >= 0; --s) {
      AncPos& e = tab[pn * TA + s];
      e.cu *= x;
      e.cq *= x;
      x *= e.alpha;
    }
    ps[pn].ep = x;
  }

  // -------------------------------------------------------------------- D -> shared (beam-major)
  __syncthreads();                                 // every warp is done reading the A tiles
  const bool have_d = mbar_wait_bounded(done, 0);
  if (!have_d) report_error(a.err, OLA_ERR_TIMEOUT, 2, t);
  tc_fence_after();
  if (have_d) {
    // M = 128: row m of D at lane m. M = 64: row m at lane (m mod 16) + 32 (m div 16), i.e.
    // the first 16 lanes of each 32-lane subpartition; the other 16 lanes of a warp read
    // unused lanes and write nothing.
    constexpr int WCOLS = NB == 128 ? R4 : DV / 2;    // columns per thread
    const int sub = warp & 3;
    const int part = warp >> 2;                       // column part of this warp
    const int pl = NB == 128 ? 32 * sub + lane : 16 * sub + (lane & 15);
    const bool writes = NB == 128 || lane < 16;
    const uint32_t ta = tmem + (uint32_t(32 * sub) << 16) + uint32_t(part * WCOLS);
#pragma unroll
    for (int c = 0; c < WCOLS / 8; ++c) {
      float yq[8], yk[8];
      tmem_ld8x2(ta + 8 * c, ta + DV + 8 * c, yq, yk);
      const int ch = (part * WCOLS + 8 * c) / 4;
      if (writes) {
        *reinterpret_cast<float4*>(ychunk(0, pl, ch)) = make_float4(yq[0], yq[1], yq[2], yq[3]);
        *reinterpret_cast<float4*>(ychunk(0, pl, ch + 1)) =
            make_float4(yq[4], yq[5], yq[6], yq[7]);
        *reinterpret_cast<float4*>(ychunk(1, pl, ch)) = make_float4(yk[0], yk[1], yk[2], yk[3]);
        *reinterpret_cast<float4*>(ychunk(1, pl, ch + 1)) =
            make_float4(yk[4], yk[5], yk[6], yk[7]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();

  // -------------------------------------------------------------------- phase 3: epilogue
  if (have_d) {
    const float* Wg = a.W;
    const int e0 = VPL * lane;                     // this lane's d_v elements
    const int ych = e0 / 4, ysub = (e0 % 4) * 4;   // chunk and byte offset in a Y row
#pragma unroll
    for (int jh = 0; jh < PPW; jh += 4) {
      float u[4][VPL], qa[4][VPL];
      VVec vv[4];
#pragma unroll
      for (int j4 = 0; j4 < 4; ++j4) {
        const int pn = p0 + jh + j4;
        const PosScal sc = ps[pn];
        vv[j4] = reinterpret_cast<const VVec*>(static_cast<const __nv_bfloat16*>(a.v) +
                                               size_t(sc.io) * DV)[lane];
        const FVec yq = *reinterpret_cast<const FVec*>(ychunk(0, pn, ych) + ysub);
        const FVec yk = *reinterpret_cast<const FVec*>(ychunk(1, pn, ych) + ysub);
        uint32_t wq[VPL], wk[VPL];
        unpack_words<VPL>(yq, wq);
        unpack_words<VPL>(yk, wk);
#pragma unroll
        for (int e = 0; e < VPL; ++e) {
          u[j4][e] = sc.ep * __uint_as_float(wk[e]);
          qa[j4][e] = sc.ep * __uint_as_float(wq[e]);
        }
      }
      constexpr int EA = 3;                        // ancestors per round
      for (int s0 = 0; s0 < n_anc; s0 += EA) {
        FVec wv[4][EA];
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
#pragma unroll
          for (int m = 0; m < EA; ++m) {
            const int s = s0 + m;
            const int row = tab[(p0 + jh + j4) * TA + (s < n_anc ? s : 0)].row;
            const FVec z = {};
            wv[j4][m] = s < n_anc ? __ldg(reinterpret_cast<const FVec*>(Wg + size_t(row) * DV) + lane)
                                  : z;
          }
        }
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
#pragma unroll
          for (int m = 0; m < EA; ++m) {
            if (s0 + m < n_anc) {
              const AncPos en = tab[(p0 + jh + j4) * TA + s0 + m];
              uint32_t ww[VPL];
              unpack_words<VPL>(wv[j4][m], ww);
#pragma unroll
              for (int e = 0; e < VPL; ++e) {
                u[j4][e] = fmaf(en.cu, __uint_as_float(ww[e]), u[j4][e]);
                qa[j4][e] = fmaf(en.cq, __uint_as_float(ww[e]), qa[j4][e]);
              }
            }
          }
        }
      }
#pragma unroll
      for (int j4 = 0; j4 < 4; ++j4) {
        const PosScal sc = ps[p0 + jh + j4];
        if (sc.b >= 0) {
          uint32_t vw[VPL / 2];
          unpack_words<VPL / 2>(vv[j4], vw);
          float ov[VPL], wn[VPL];
#pragma unroll
          for (int e = 0; e < VPL; ++e) {
            const float vf = (e & 1) ? bfh(vw[e / 2]) : bfl(vw[e / 2]);
            wn[e] = sc.beta * (vf - sc.alpha * u[j4][e]);
            ov[e] = fmaf(sc.alpha, qa[j4][e], sc.c0 * wn[e]);
          }
          FVec ob, wb;
          uint32_t* op = reinterpret_cast<uint32_t*>(&ob);
          uint32_t* wp = reinterpret_cast<uint32_t*>(&wb);
#pragma unroll
          for (int e = 0; e < VPL; ++e) {
            op[e] = __float_as_uint(ov[e]);
            wp[e] = __float_as_uint(wn[e]);
          }
          reinterpret_cast<FVec*>(a.o + size_t(sc.io) * DV)[lane] = ob;
          reinterpret_cast<FVec*>(a.W + size_t(sc.wnew) * DV)[lane] = wb;
        }
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L.ncols);
  }
}

constexpr int kPosCtaBeams = 64;       // beams per CTA of the dispatched variant

size_t replay_pos_smem(int d_k, int d_v, int T_max) {
  return pos_layout(d_k, d_v, T_max, kPosCtaBeams).bytes;
}

cudaError_t launch_plan(const StepArgs& a, cudaStream_t stream);

template <int DK, int DV, int NB>
static cudaError_t launch_pos_t(const CUtensorMap& mhi, const CUtensorMap& mlo,
                                const StepArgs& a, cudaStream_t stream) {
  const PosLayout L = pos_layout(DK, DV, a.T_max, NB);
  const unsigned grid = unsigned(a.R) * a.H * ((a.B + NB - 1) / NB);
  auto kern = replay_pos_kernel<DK, DV, NB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(L.bytes));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  kern<<<grid, NB * 4, L.bytes, stream>>>(mhi, mlo, a);
  return cudaGetLastError();
}

bool replay_pos_supported(int d_k, int d_v) { return d_k <= 128 && d_v <= 128; }

cudaError_t launch_replay_pos(const StepArgs& a, const CUtensorMap& mhi, const CUtensorMap& mlo,
                              cudaStream_t stream) {
  cudaError_t e = launch_plan(a, stream);
  if (e != cudaSuccess) return e;
  constexpr int NB = kPosCtaBeams;
  if (a.d_k == 64 && a.d_v == 64) return launch_pos_t<64, 64, NB>(mhi, mlo, a, stream);
  if (a.d_k == 64 && a.d_v == 128) return launch_pos_t<64, 128, NB>(mhi, mlo, a, stream);
  if (a.d_k == 128 && a.d_v == 64) return launch_pos_t<128, 64, NB>(mhi, mlo, a, stream);
  if (a.d_k == 128 && a.d_v == 128) return launch_pos_t<128, 128, NB>(mhi, mlo, a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ola
