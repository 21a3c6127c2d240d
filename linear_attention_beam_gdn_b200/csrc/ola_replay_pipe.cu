// Projection-replay decode step: persistent, pipelined, state-major (sm_100a; d_v = 128,
// d_k = 64 or 128, T_max <= 12, bf16 inputs).
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
// Work unit: one (request, head) and 32 consecutive depth-first positions (ola_plan.cu). One
// CTA per SM walks a contiguous range of units through a three-stage ring, so the loads of
// the next units run under the arithmetic of the current one. Warp roles:
//   warps 0-2  producers: read the unit's beams and parent chains, find the distinct ancestor
//              records of each chain slot (depth-first order makes equal records adjacent),
//              and copy with cp.async the q, k rows (into the 128-byte swizzled MMA operand
//              layout), the v rows, and the key and w rows of up to 56 distinct ancestors.
//   warp 3     MMA: D[i][p] = sum_k S[i][k] x_p[k] on tcgen05, state-major (M = d_v = 128
//              state rows, N = 32 positions); S_ctx (bf16 hi + lo) is the A operand held in
//              tensor memory, the staged q / k tiles are B. One accumulator per stage.
//   warps 4-7  chain: load S_ctx into tensor memory when the (request, head) changes, then
//              the dot products k_j . k_t, k_j . q_t (warp-level MMA over the staged keys),
//              k_t . q_t, the decay products, and the appends (k_t row, alpha_t, chain row).
//   warps 8-15 epilogue: thread = state row i; per position reads D from tensor memory, adds
//              the ancestors' w_j[i] (staged rows, else global), forms w_t[i] and o_t[i] and
//              stores them (a warp writes 128 contiguous bytes of one row).
// Every wait is bounded; on timeout the kernel records OLA_ERR_TIMEOUT and finishes.
#include "ola_device.cuh"

namespace ola {

constexpr int kPipeNB = 32;      // depth-first positions per unit (MMA N)
constexpr int kPipeUCap = 56;    // distinct ancestor records staged per unit
constexpr int kPipeStages = 3;
constexpr int kPipeMaxT = 12;    // largest T_max this kernel takes
constexpr int kPipeProd = 3;     // producer warps
constexpr int kPipeWarps = kPipeProd + 1 + 4 + 8;
constexpr int kPipeDV = 128;

struct PipeAnc {                 // one (position, chain slot) entry, 16 bytes
  int ref;                       // -(u+1): staged ancestor u of the unit; else its record row
  float cu, cq;                  // d_j (k_j . k_t), d_j (k_j . q_t)
  int woff;                      // byte offset of its staged w row (the zero row if unstaged)
};

struct PipeScal {                // per-position scalars, 32 bytes
  int io, wnew, b, ovf;          // input/output row, record row of w_t, beam (-1: no beam),
                                 // (position 0) 1 if some ancestor of the unit is unstaged
  float ep, alpha, beta, c0;
};

// Shared memory of one stage (every block 1024-byte aligned):
//   X [slice][q | k][32 rows][128 B]   128-byte swizzled (MMA operand B)
//   K [slice][56 rows][128 B]          staged ancestor keys, same swizzle
//   W [57 rows][d_v] fp32              staged ancestor w rows, then a row of zeros
//   V [32 rows][d_v] bf16
struct PipeLayout {
  int NSL, TA;
  uint32_t xs, ks, k_off, w_off, v_off, stage;
  size_t tab_off, ps_off, gb_off, al_off, list_off, bar_off, bytes;
};

__host__ __device__ inline PipeLayout pipe_layout(int d_k, int T_max) {
  PipeLayout L;
  L.NSL = d_k / 64;
  L.TA = T_max > 1 ? T_max - 1 : 1;
  L.xs = uint32_t(kPipeNB) * 128u;                         // one (slice, side) tile
  L.ks = uint32_t(kPipeUCap) * 128u;                       // one slice of staged keys
  L.k_off = uint32_t(L.NSL) * 2u * L.xs;
  L.w_off = L.k_off + uint32_t(L.NSL) * L.ks;
  L.v_off = L.w_off + uint32_t(kPipeUCap + 1) * kPipeDV * 4u;
  L.stage = (L.v_off + uint32_t(kPipeNB) * kPipeDV * 2u + 1023u) & ~1023u;  // swizzle atoms
  L.tab_off = size_t(kPipeStages) * L.stage;
  L.ps_off = L.tab_off + size_t(kPipeStages) * sizeof(PipeAnc) * kPipeNB * L.TA;
  L.gb_off = L.ps_off + size_t(kPipeStages) * sizeof(PipeScal) * kPipeNB;   // (g, beta)
  L.al_off = L.gb_off + size_t(kPipeStages) * 8 * kPipeNB;       // alpha of staged ancestors
  L.list_off = L.al_off + size_t(kPipeStages) * 4 * kPipeUCap;   // record rows, per producer
  L.bar_off = L.list_off + size_t(kPipeStages) * kPipeProd * 4 * kPipeUCap;
  L.bytes = L.bar_off + 128 + 1024;                        // barriers, holder, alignment
  return L;
}


template <int DK>
__global__ void __launch_bounds__(kPipeWarps * 32, 1)
replay_pipe_kernel(const __nv_bfloat16* __restrict__ S_hi, const __nv_bfloat16* __restrict__ S_lo,
                   StepArgs a) {
  constexpr int NB = kPipeNB, UC = kPipeUCap, DV = kPipeDV, NS = kPipeStages;
  constexpr int NSL = DK / 64, CPL = DK / 32;
  constexpr int CR = DK / 8;       // 16-byte chunks of a key row
  constexpr int RPI = 32 / CR;     // key rows copied per warp instruction
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align_smem_1024(smem_raw);
  const PipeLayout L = pipe_layout(DK, a.T_max);
  const int TA = L.TA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* full = bars;              // [NS] stage loaded: 32 x 4 cp.async arrivals + 1
  uint64_t* empty = bars + NS;        // [NS] stage consumed: MMA commit + 4 chain + 8 epilogue
  uint64_t* dfull = bars + 2 * NS;    // [NS] accumulators of the stage's unit ready
  uint64_t* cdone = bars + 3 * NS;    // [NS] chain warps done with the stage's unit
  uint64_t* sready = bars + 4 * NS;   // [2]  S_ctx buffer loaded into tensor memory
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 4 * NS + 2);
  auto stage = [&](int s) { return smem + size_t(s) * L.stage; };
  auto tab = [&](int s) {
    return reinterpret_cast<PipeAnc*>(smem + L.tab_off) + size_t(s) * NB * TA;
  };
  auto psc = [&](int s) { return reinterpret_cast<PipeScal*>(smem + L.ps_off) + s * NB; };
  auto lst = [&](int s) {
    return reinterpret_cast<int*>(smem + L.list_off) + s * kPipeProd * UC;
  };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = a.t, n_anc = t - 1;
  const int n_chunks = (a.B + NB - 1) / NB;
  const int n_units = a.R * a.H * n_chunks;
  const int ubeg = int((long long)blockIdx.x * n_units / gridDim.x);
  const int n_my = int((long long)(blockIdx.x + 1) * n_units / gridDim.x) - ubeg;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 32 * kPipeProd + 1);
      mbar_init(&empty[s], 1 + 4 + 8);
      mbar_init(&dfull[s], 1);
      mbar_init(&cdone[s], 4);
    }
    mbar_init(&sready[0], 4);
    mbar_init(&sready[1], 4);
    fence_barrier_init();
  }
  if (warp == kPipeProd) tmem_alloc(holder, 512);
  for (int x = tid; x < NS * DV; x += blockDim.x)   // the zero w row of each stage
    reinterpret_cast<float*>(stage(x / DV) + L.w_off + UC * DV * 4)[x % DV] = 0.f;
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;   // columns [0,192): accumulators, [256,512): S_ctx buffers

  if (warp < kPipeProd) {
    // ------------------------------------------------------------------ producers
    // Every producer warp reads the unit's beams and chains and finds the same distinct
    // records; warp pw copies its share (row groups and records with index = pw mod 3).
    // Warp 0 also writes the per-position table and scalars.
    const int pw = warp;
    const unsigned char* qg = static_cast<const unsigned char*>(a.q);
    const unsigned char* kg = static_cast<const unsigned char*>(a.k);
    const unsigned char* vg = static_cast<const unsigned char*>(a.v);
    const unsigned char* krg = static_cast<const unsigned char*>(a.Kr);
    const unsigned char* wg = reinterpret_cast<const unsigned char*>(a.W);
    const unsigned le = kFull >> (31 - lane);
    int issued = 0;
    for (int i = 0; i < n_my; ++i) {
      const int u = ubeg + i, s = i % NS, n = i / NS;
      const int rh = u / n_chunks, c0 = (u % n_chunks) * NB;
      const int r = rh / a.H, h = rh % a.H;
      if (i >= NS && !__all_sync(kFull, mbar_wait_bounded(&empty[s], (n - 1) & 1))) {
        if (lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 10, t);
        break;
      }
      PipeScal* ps = psc(s);
      PipeAnc* tb = tab(s);
      int* list = lst(s) + pw * UC;
      unsigned char* st = stage(s);
      // lane = position (past the last beam: the last beam again, flagged b = -1)
      const int pos = c0 + lane;
      const int pc = pos < a.B ? pos : a.B - 1;
      const int b = a.perm[size_t(r) * a.B + pc];
      const int io = (r * a.B + b) * a.H + h;
      int ch[kPipeMaxT - 1];
#pragma unroll
      for (int sl = 0; sl < kPipeMaxT - 1; ++sl)
        ch[sl] = sl < n_anc ? a.pchain[(size_t(r) * a.B + pc) * a.T_max + sl] : 0;
      if (pw == 0) {
        PipeScal sc;
        sc.io = io;
        sc.wnew = int(rec_index(a, t - 1, r, h, b));
        sc.b = pos < a.B ? b : -1;
        sc.ovf = 0;
        sc.ep = 1.f;
        sc.alpha = 0.f;
        sc.beta = 0.f;
        sc.c0 = 0.f;
        ps[lane] = sc;
        if (h == 0 && pos < a.B) {                  // chain row of the new beam (head 0 only)
          const size_t crow = chain_row(a, t - 1, r, b);
#pragma unroll
          for (int sl = 0; sl < kPipeMaxT - 1; ++sl)
            if (sl < n_anc) a.C[crow + sl] = ch[sl];
          a.C[crow + n_anc] = b;
        }
        float* gb = reinterpret_cast<float*>(smem + L.gb_off) + size_t(s) * 2 * NB;
        cp_async4(gb + 2 * lane, a.g + io);
        cp_async4(gb + 2 * lane + 1, a.beta + io);
      }
      // q, k rows into the swizzled operand tiles (RPI rows per instruction)
      for (int it = pw; it < NB / RPI; it += kPipeProd) {
        const int p = it * RPI + lane / CR, c = lane % CR;
        const int iop = __shfl_sync(kFull, io, p);
        const size_t go = size_t(iop) * DK * 2 + size_t(c) * 16;
        const uint32_t xo = uint32_t(p) * 128u + uint32_t(((c & 7) ^ (p & 7)) << 4);
        cp_async16(st + ((c >> 3) * 2) * L.xs + xo, qg + go);
        cp_async16(st + ((c >> 3) * 2 + 1) * L.xs + xo, kg + go);
      }
      // v rows (256 bytes: two rows per instruction)
      for (int it = pw; it < NB / 2; it += kPipeProd) {
        const int p = it * 2 + (lane >> 4), c = lane & 15;
        const int iop = __shfl_sync(kFull, io, p);
        cp_async16(st + L.v_off + p * (DV * 2) + c * 16, vg + size_t(iop) * DV * 2 + c * 16);
      }
      // distinct records per chain slot: equal records are adjacent, so a record is new where
      // it differs from the previous position's; u = running count of new records
      int ubase = 0;
#pragma unroll
      for (int sl = 0; sl < kPipeMaxT - 1; ++sl) {
        if (sl < n_anc) {
          const int e = ch[sl];
          const int prev = __shfl_up_sync(kFull, e, 1);
          const bool f = lane == 0 || e != prev;
          const unsigned m = __ballot_sync(kFull, f);
          const int uu = ubase + __popc(m & le) - 1;
          const int row = int(rec_index(a, sl, r, h, e));
          if (pw == 0) tb[lane * TA + sl].ref = uu < UC ? -(uu + 1) : row;
          if (f && uu < UC) list[uu] = row;
          ubase += __popc(m);
        }
      }
      const int U = ubase < UC ? ubase : UC;
      if (pw == 0 && lane == 0) ps[0].ovf = ubase > UC ? 1 : 0;
      __syncwarp();
      for (int it = pw; it * RPI < U; it += kPipeProd) {   // staged keys, same swizzle as X
        const int uu = it * RPI + lane / CR, c = lane % CR;
        if (uu < U)
          cp_async16(st + L.k_off + (c >> 3) * L.ks + uu * 128 + (((c & 7) ^ (uu & 7)) << 4),
                     krg + size_t(list[uu]) * DK * 2 + size_t(c) * 16);
      }
      for (int uu = pw; uu < U; uu += kPipeProd)           // staged w rows (512 bytes)
        cp_async16(st + L.w_off + uu * (DV * 4) + lane * 16,
                   wg + size_t(list[uu]) * DV * 4 + size_t(lane) * 16);
      if (pw == 0) {                                       // their alphas
        float* al = reinterpret_cast<float*>(smem + L.al_off) + size_t(s) * UC;
        for (int uu = lane; uu < U; uu += 32) cp_async4(al + uu, a.A + list[uu]);
      }
      cp_async_arrive(&full[s]);
      __syncwarp();
      if (pw == 0 && lane == 0) mbar_arrive(&full[s]);
      issued = i + 1;
    }
    // the CTA may not exit with copies in flight
    for (int i = issued > NS ? issued - NS : 0; i < issued; ++i)
      mbar_wait_bounded(&full[i % NS], (i / NS) & 1);
  } else if (warp == kPipeProd) {
    // ------------------------------------------------------------------ MMA (lane 0)
    int sver = -1, prev_rh = -1, last = -1;
    bool ok = true;
    for (int i = 0; i < n_my && ok; ++i) {
      const int u = ubeg + i, s = i % NS, n = i / NS, rh = u / n_chunks;
      if (rh != prev_rh) {
        ++sver;
        prev_rh = rh;
      }
      const int j = sver & 1;
      if (lane == 0) {
        ok = mbar_wait_bounded(&full[s], n & 1) && mbar_wait_bounded(&sready[j], (sver >> 1) & 1);
        if (ok) {
          tc_fence_after();
          const uint32_t d = tmem + uint32_t(s) * 2u * NB;
          const uint32_t sa = tmem + 256u + uint32_t(j) * 128u;
          const uint32_t idesc = idesc_bf16_f32(128, NB);
          const unsigned char* st = stage(s);
#pragma unroll
          for (int ks = 0; ks < NSL; ++ks) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const int kstep = ks * 4 + kk;
              const uint64_t bq = sw128_kmajor_desc(smem_u32(st + (ks * 2) * L.xs) + kk * 32);
              const uint64_t bk = sw128_kmajor_desc(smem_u32(st + (ks * 2 + 1) * L.xs) + kk * 32);
              const uint32_t ahi = sa + kstep * 8, alo = sa + DK / 2 + kstep * 8;
              const uint32_t acc = kstep != 0 ? 1u : 0u;
              umma_bf16_ts(d, ahi, bq, idesc, acc);
              umma_bf16_ts(d, alo, bq, idesc, 1u);
              umma_bf16_ts(d + NB, ahi, bk, idesc, acc);
              umma_bf16_ts(d + NB, alo, bk, idesc, 1u);
            }
          }
          umma_commit(&dfull[s]);
          umma_commit(&empty[s]);
          last = i;
        } else {
          report_error(a.err, OLA_ERR_TIMEOUT, 11, t);
        }
      }
      ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
    }
    // tensor memory is released only once the last MMA has completed
    if (lane == 0 && last >= 0) mbar_wait_bounded(&dfull[last % NS], (last / NS) & 1);
    __syncwarp();
  } else if (warp < kPipeProd + 5) {
    // ------------------------------------------------------------------ chain warps
    const int cw = warp - (kPipeProd + 1), sp = warp & 3;
    const int gq = lane >> 2, c4 = lane & 3;
    const int p = 8 * cw + gq;                        // this lane's position in the MMA
    int sver = -1, prev_rh = -1;
    __nv_bfloat16* kout = static_cast<__nv_bfloat16*>(a.Kr);
    const __nv_bfloat16* krec = kout;
    for (int i = 0; i < n_my; ++i) {
      const int u = ubeg + i, s = i % NS, n = i / NS;
      const int rh = u / n_chunks;
      const bool new_s = rh != prev_rh;
      if (new_s) {
        ++sver;
        prev_rh = rh;
      }
      bool ok = mbar_wait_bounded(&full[s], n & 1);
      // a new S_ctx overwrites the buffer of version sver - 2, whose last unit is at most
      // i - 2: its MMAs (completed in order) must be done
      if (new_s && i >= 2) ok = ok && mbar_wait_bounded(&dfull[(i - 2) % NS], ((i - 2) / NS) & 1);
      if (!__all_sync(kFull, ok)) {
        if (lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 12, t);
        break;
      }
      if (new_s) {
        // S_ctx rows 32 sp .. 32 sp + 31 (hi, then lo) into buffer sver & 1; one row per lane,
        // two bf16 per 32-bit column, lower k in the low half (memory order)
        tc_fence_after();
        const int j = sver & 1;
        const int row = 32 * sp + lane;
        const uint32_t ta = tmem + (uint32_t(32 * sp) << 16) + 256u + uint32_t(j) * 128u;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint4* src = reinterpret_cast<const uint4*>((half ? S_lo : S_hi) +
                                                            (size_t(rh) * 128 + row) * DK);
          uint4 v[DK / 8];
#pragma unroll
          for (int c = 0; c < DK / 8; ++c) v[c] = __ldg(src + c);
#pragma unroll
          for (int c = 0; c < DK / 32; ++c) {
            const uint4 w4[4] = {v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]};
            tmem_st16(ta + half * (DK / 2) + c * 16, w4);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sready[j]);
      }
      const unsigned char* st = stage(s);
      PipeScal* ps = psc(s);
      PipeAnc* tb = tab(s);
      const float* alst = reinterpret_cast<const float*>(smem + L.al_off) + size_t(s) * UC;
      const float* gb = reinterpret_cast<const float*>(smem + L.gb_off) + size_t(s) * 2 * NB;
      // Dot products on warp-level MMA (m16n8k16): A rows 0-7 = keys of chain slot sl of the 8
      // positions, rows 8-15 = slot sl+1; B columns = the positions' k_t (then q_t); only the
      // diagonal is used. The k index is permuted identically in A and B so that lane (g, c)
      // reads whole 16-byte chunks: chunk m of a row = elements [32 m + 8 c, +8).
      uint4 xq[CPL], xk[CPL];
      float c0p = 0.f;
#pragma unroll
      for (int m = 0; m < CPL; ++m) {
        const int e = 32 * m + 8 * c4, ks = e >> 6, chn = (e & 63) >> 3;
        const uint32_t off = uint32_t(p) * 128u + uint32_t((chn ^ (p & 7)) << 4);
        xq[m] = *reinterpret_cast<const uint4*>(st + (ks * 2) * L.xs + off);
        xk[m] = *reinterpret_cast<const uint4*>(st + (ks * 2 + 1) * L.xs + off);
        c0p += dot8_bf16(xk[m], xq[m]);
      }
      c0p += __shfl_xor_sync(kFull, c0p, 1);
      c0p += __shfl_xor_sync(kFull, c0p, 2);
      if (c4 == 0) ps[p].c0 = c0p;
      {  // append k_t to the key records
        const int b = ps[p].b;
        const int wnew = ps[p].wnew;
        if (b >= 0) {
#pragma unroll
          for (int m = 0; m < CPL; ++m)
            *reinterpret_cast<uint4*>(kout + size_t(wnew) * DK + 32 * m + 8 * c4) = xk[m];
        }
      }
      for (int s0 = 0; s0 < n_anc; s0 += 2) {
        uint4 kr[2][CPL];
#pragma unroll
        for (int i2 = 0; i2 < 2; ++i2) {
          const int sl = s0 + i2 < n_anc ? s0 + i2 : s0;
          const int ref = tb[p * TA + sl].ref;
          if (ref < 0) {
            const int uu = -ref - 1;
#pragma unroll
            for (int m = 0; m < CPL; ++m) {
              const int e = 32 * m + 8 * c4, ks = e >> 6, chn = (e & 63) >> 3;
              kr[i2][m] = *reinterpret_cast<const uint4*>(st + L.k_off + ks * L.ks + uu * 128 +
                                                          ((chn ^ (uu & 7)) << 4));
            }
          } else {
            const uint4* src = reinterpret_cast<const uint4*>(krec + size_t(ref) * DK + 8 * c4);
#pragma unroll
            for (int m = 0; m < CPL; ++m) kr[i2][m] = __ldg(src + 4 * m);
          }
        }
        float dk[4] = {0.f, 0.f, 0.f, 0.f}, dq[4] = {0.f, 0.f, 0.f, 0.f};
        float ek[4] = {0.f, 0.f, 0.f, 0.f}, eq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int m = 0; m < CPL; ++m) {                // two accumulators per side: shorter chains
          mma_16816_bf16(dk, kr[0][m].x, kr[1][m].x, kr[0][m].y, kr[1][m].y, xk[m].x, xk[m].y);
          mma_16816_bf16(dq, kr[0][m].x, kr[1][m].x, kr[0][m].y, kr[1][m].y, xq[m].x, xq[m].y);
          mma_16816_bf16(ek, kr[0][m].z, kr[1][m].z, kr[0][m].w, kr[1][m].w, xk[m].z, xk[m].w);
          mma_16816_bf16(eq, kr[0][m].z, kr[1][m].z, kr[0][m].w, kr[1][m].w, xq[m].z, xq[m].w);
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          dk[x] += ek[x];
          dq[x] += eq[x];
        }
        if (c4 == (gq >> 1)) {                       // this lane holds D[gq][gq], D[8+gq][gq]
          const int o = gq & 1;
          tb[p * TA + s0].cu = dk[o];
          tb[p * TA + s0].cq = dq[o];
          if (s0 + 1 < n_anc) {
            tb[p * TA + s0 + 1].cu = dk[2 + o];
            tb[p * TA + s0 + 1].cq = dq[2 + o];
          }
        }
      }
      __syncwarp();
      if (lane < 8) {                                 // decay products and per-position scalars
        const int pd = 8 * cw + lane;
        const int b = ps[pd].b, wnew = ps[pd].wnew;
        float al[kPipeMaxT - 1];
#pragma unroll
        for (int sl = 0; sl < kPipeMaxT - 1; ++sl) {
          al[sl] = 1.f;
          if (sl < n_anc) {
            const int ref = tb[pd * TA + sl].ref;
            al[sl] = ref < 0 ? alst[-ref - 1] : a.A[ref];
          }
        }
        const float gt = gb[2 * pd], bt = gb[2 * pd + 1];
        float x = 1.f;
#pragma unroll
        for (int sl = kPipeMaxT - 2; sl >= 0; --sl) {
          if (sl < n_anc) {
            PipeAnc& e = tb[pd * TA + sl];
            e.cu *= x;
            e.cq *= x;
            e.woff = (e.ref < 0 ? -e.ref - 1 : UC) * (DV * 4);
            x *= al[sl];
          }
        }
        const float alpha = expf(gt);
        ps[pd].ep = x;
        ps[pd].alpha = alpha;
        ps[pd].beta = bt;
        if (b >= 0) a.A[wnew] = alpha;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&cdone[s]);
        mbar_arrive(&empty[s]);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps
    // thread = state row i (tensor-memory lane); warp (sp, ph) = rows 32 sp.., positions 16 ph..
    const int ew = warp - (kPipeProd + 5), sp = warp & 3, ph = ew >> 2;
    const int row = 32 * sp + lane;
    const uint32_t tl = tmem + (uint32_t(32 * sp) << 16);
    for (int i = 0; i < n_my; ++i) {
      const int s = i % NS, n = i / NS;
      bool ok = mbar_wait_bounded(&dfull[s], n & 1);
      ok = ok && mbar_wait_bounded(&cdone[s], n & 1);
      if (!__all_sync(kFull, ok)) {
        if (lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 13, t);
        break;
      }
      tc_fence_after();
      const unsigned char* st = stage(s);
      const __nv_bfloat16* Vs = reinterpret_cast<const __nv_bfloat16*>(st + L.v_off);
      const PipeScal* ps = psc(s);
      const PipeAnc* tb = tab(s);
      const bool ovf = ps[0].ovf != 0;
#pragma unroll 1
      for (int pb = 0; pb < 2; ++pb) {
        const int p0 = 16 * ph + 8 * pb;
        float dq[8], dk[8];
        tmem_ld8x2(tl + uint32_t(s) * 2u * NB + p0, tl + uint32_t(s) * 2u * NB + NB + p0, dq, dk);
        float yk[8], yq[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float ep = ps[p0 + j].ep;
          yk[j] = ep * dk[j];
          yq[j] = ep * dq[j];
        }
        // staged ancestors (unstaged ones point at the zero row here)
        const unsigned char* wrow = st + L.w_off + row * 4;
        for (int sl = 0; sl < n_anc; ++sl) {
          float4 e[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) e[j] = *reinterpret_cast<const float4*>(&tb[(p0 + j) * TA + sl]);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float w = *reinterpret_cast<const float*>(wrow + __float_as_int(e[j].w));
            yk[j] = fmaf(e[j].y, w, yk[j]);
            yq[j] = fmaf(e[j].z, w, yq[j]);
          }
        }
        if (ovf) {                                   // ancestors past the staging capacity
          for (int sl = 0; sl < n_anc; ++sl) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 e = *reinterpret_cast<const float4*>(&tb[(p0 + j) * TA + sl]);
              const int ref = __float_as_int(e.x);
              if (ref >= 0) {
                const float w = __ldg(a.W + size_t(ref) * DV + row);
                yk[j] = fmaf(e.y, w, yk[j]);
                yq[j] = fmaf(e.z, w, yq[j]);
              }
            }
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const PipeScal sc = ps[p0 + j];
          if (sc.b >= 0) {
            const float v = __bfloat162float(Vs[(p0 + j) * DV + row]);
            const float wn = sc.beta * (v - sc.alpha * yk[j]);
            const float o = fmaf(sc.alpha, yq[j], sc.c0 * wn);
            a.o[size_t(sc.io) * DV + row] = o;
            a.W[size_t(sc.wnew) * DV + row] = wn;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kPipeProd) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------- host side

bool replay_pipe_supported(int d_k, int d_v, int T_max) {
  return d_v == kPipeDV && (d_k == 64 || d_k == 128) && T_max <= kPipeMaxT;
}

size_t replay_pipe_smem(int d_k, int T_max) { return pipe_layout(d_k, T_max).bytes; }

cudaError_t launch_plan(const StepArgs& a, cudaStream_t stream);

template <int DK>
static cudaError_t launch_pipe_t(const void* S_hi, const void* S_lo, const StepArgs& a, int n_sm,
                                 cudaStream_t stream) {
  const PipeLayout L = pipe_layout(DK, a.T_max);
  const long long n_units = (long long)a.R * a.H * ((a.B + kPipeNB - 1) / kPipeNB);
  const unsigned grid = unsigned(n_units < n_sm ? n_units : n_sm);
  auto kern = replay_pipe_kernel<DK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(L.bytes));
  if (e != cudaSuccess) return e;
  kern<<<grid, kPipeWarps * 32, L.bytes, stream>>>(static_cast<const __nv_bfloat16*>(S_hi),
                                                   static_cast<const __nv_bfloat16*>(S_lo), a);
  return cudaGetLastError();
}

// S_hi, S_lo: the shared state split into bf16 hi + lo, [R*H][128][d_k].
cudaError_t launch_replay_pipe(const StepArgs& a, const void* S_hi, const void* S_lo,
                               cudaStream_t stream) {
  cudaError_t e = launch_plan(a, stream);
  if (e != cudaSuccess) return e;
  int dev = 0, n_sm = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (a.d_k == 64) return launch_pipe_t<64>(S_hi, S_lo, a, n_sm, stream);
  if (a.d_k == 128) return launch_pipe_t<128>(S_hi, S_lo, a, n_sm, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ola
