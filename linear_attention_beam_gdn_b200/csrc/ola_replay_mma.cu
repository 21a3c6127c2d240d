// Projection-replay decode step with both contractions on tensor cores: persistent, pipelined,
// state-major (sm_100a; d_v = 128, d_k = 64 or 128, T_max <= 12, B <= 1024, bf16 inputs).
//
// Mathematics ("Scientific Impact Assessment: OneLA", §1 Core Contribution: one shared
// post-prefill state, append-only transition records, projection replay through the key and
// query contractions, one fused kernel reusing the shared state across beams). For the beam at
// depth-first position p with parent chain j = 1..t-1 (records w_j, k_j, alpha_j):
//     u_p = e_p S_ctx k_p + sum_j d_pj (k_j . k_p) w_j,    w_p = beta_p (v_p - alpha_p u_p)
//     o_p = alpha_p (e_p S_ctx q_p + sum_j d_pj (k_j . q_p) w_j) + (k_p . q_p) w_p
// with d_pj = prod_{i>j} alpha_i along p's chain and e_p = prod_j alpha_j.
//
// Work unit: one (request, head) and one unit of at most 32 consecutive depth-first positions
// whose chains reach at most 48 distinct records u (plan_units_kernel). For the unit,
//     D1[i][x]  = sum_k S_ctx[i][k] x[k]               x = q_p, k_p          (tcgen05, M = 128)
//     G[x][u]   = x . k_u                                                    (tcgen05, M = 64)
//     Cf[x][u]  = d_pu G[x][u]  (zero where u is not on p's chain)
//     D2[i][x]  = sum_u w_u[i] Cf[x][u]                                      (tcgen05, M = 128)
// so u_p[i] = e_p D1[i][k_p] + D2[i][k_p] and the query side likewise. The w records are kept as
// two bf16 planes (hi = bf16(w), lo = bf16(w - hi)); S_ctx is split the same way at create, and
// Cf too, so each product runs as hi*hi + lo*hi + hi*lo with fp32 accumulation (the "bf16x2"
// split of Henry, Tang & Heinecke 2019).
//
// One CTA per SM walks the units of its (request, head) pairs, dealt round-robin, through a
// three-stage ring. Warp roles:
//   warps 0-5   producers: TMA row gathers (tile::gather4, 128-byte swizzle) of the unit's q, k
//               and v rows, distinct ancestor keys and w records (the latter as the MN-major
//               operand), one list of copies dealt out in six chunks; cp.async of the
//               per-position scalars.
//   warp 6      MMA: G with the staged q, k tile as A and the ancestor keys as B; D1 with S_ctx
//               (bf16 hi + lo) held in tensor memory as the A operand; D2 with the staged w
//               planes as the A operand and Cf as B, written over G. Two accumulator stages;
//               D2 of unit i - 1 is issued before G and D1 of unit i.
//   warp 7      prep: decay table, k_p . q_p, per-position scalars, appends of k_p and alpha_p.
//   warps 8-11  coefficients: S_ctx into tensor memory when the (request, head) changes; Cf
//               from G and the decay table.
//   warps 12-19 epilogue: thread = state row i; w_p[i] and o_p[i] from D1, D2 and the scalars;
//               stores o (fp32) and the w record (hi, lo).
// Every wait is bounded; on timeout the kernel records OLA_ERR_TIMEOUT and finishes.
#include "ola_device.cuh"

namespace ola {

constexpr int kMmaStages = 3;
constexpr int kMmaMaxT = 12;
constexpr int kMmaMaxB = 1024;
constexpr int kMmaDV = 128;
// A TMA instruction holds its warp for several hundred cycles plus roughly eighty per active
// lane, while the instructions of different warps proceed in parallel: the copies of a unit are
// spread over six producer warps, one warp-wide gather instruction each.
constexpr int kMmaProd = 6, kMmaCoef = 4, kMmaEpi = 8;
constexpr int kMmaWarps = kMmaProd + 2 + kMmaCoef + kMmaEpi;   // 20 warps, 5 per subpartition
constexpr int kMmaWMma = kMmaProd;              // warp 6
constexpr int kMmaWPrep = kMmaProd + 1;         // warp 7
constexpr int kMmaWCoef = kMmaProd + 2;         // warps 8..11 (subpartitions 0..3)
constexpr int kMmaWEpi = kMmaWCoef + kMmaCoef;  // warps 12..19
static_assert(kMmaWCoef % 4 == 0 && kMmaWEpi % 4 == 0, "tensor-memory lane quarters follow warp % 4");

// Record row of (step slot, request r, beam b, head h) in this kernel's record storage, which
// keeps the heads of a beam next to each other: [T_max][R][B][H] (the heads of one beam are
// decoded at about the same time by neighbouring CTAs, so their rows share DRAM pages).
__device__ __forceinline__ int rec_row_hm(const StepArgs& a, int slot, int r, int h, int b) {
  return ((slot * a.R + r) * a.B + b) * a.H + h;
}

struct MmaInfo {                 // per stage
  int r, h, start, n_pos;
  int U, first, last, pad;
  int beam[kUnitPos];
  float gb[2 * kUnitPos];        // (g, beta) of each position
  float alpha[kUnitAnc];         // alpha of each distinct record
  uint8_t upos[kUnitPos][16];    // record index u of each (position, chain slot)
};

struct MmaScal {                 // per position
  float e, alpha, beta, c0;
  int io, wnew, valid, pad;
};

// Shared memory (every tile 1024-byte aligned):
//   stage s: X [NSL][64 rows: q of positions 0-31 | k of positions 0-31][128 B]  K-major, sw128
//            KA [NSL][48 rows][128 B]       ancestor keys, same swizzle
//            WH, WL [6 groups of 8 records][2 halves of d_v][8][128 B]  MN-major, sw128
//            V [2 halves of d_v][32 positions][128 B]  sw128, MmaInfo
//   then CH, CL [64 rows][128 B] (Cf hi, lo; K-major, sw128), DEC [2][32][48] fp32,
//   SC [2][32], barriers.
struct MmaLayout {
  uint32_t ka_off, wh_off, wl_off, v_off, info_off, stage;
  uint32_t ch_off, cl_off, dec_off, sc_off, bar_off, bytes;
};

__host__ __device__ inline MmaLayout mma_layout(int d_k) {
  const uint32_t NSL = uint32_t(d_k) / 64u;
  MmaLayout L;
  L.ka_off = NSL * 8192u;
  L.wh_off = L.ka_off + NSL * uint32_t(kUnitAnc) * 128u;
  L.wl_off = L.wh_off + uint32_t(kUnitAnc / 8) * 2048u;
  L.v_off = L.wl_off + uint32_t(kUnitAnc / 8) * 2048u;
  L.info_off = L.v_off + uint32_t(kUnitPos) * kMmaDV * 2u;
  L.stage = (L.info_off + uint32_t(sizeof(MmaInfo)) + 1023u) & ~1023u;
  L.ch_off = uint32_t(kMmaStages) * L.stage;
  L.cl_off = L.ch_off + 8192u;
  L.dec_off = L.cl_off + 8192u;
  L.sc_off = L.dec_off + 2u * kUnitPos * kUnitAnc * 4u;
  L.bar_off = L.sc_off + 2u * kUnitPos * uint32_t(sizeof(MmaScal));
  L.bytes = L.bar_off + 256u + 1024u;
  return L;
}

template <int DK>
__global__ void __launch_bounds__(kMmaWarps * 32, 1)
replay_mma_kernel(const __nv_bfloat16* __restrict__ S_hi, const __nv_bfloat16* __restrict__ S_lo,
                  StepArgs a, UnitPlan up, const __grid_constant__ CUtensorMap mq,
                  const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                  const __grid_constant__ CUtensorMap mkr, const __grid_constant__ CUtensorMap mw) {
  constexpr int NS = kMmaStages, DV = kMmaDV, UC = kUnitAnc, NP = kUnitPos;
  constexpr int CR = DK / 8;       // 16-byte chunks of a key row
  constexpr int NSL = DK / 64;     // 64-column slices of a key row
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align_smem_1024(smem_raw);
  const MmaLayout L = mma_layout(DK);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* full = bars;             // [NS] stage loaded: cp.async arrivals + 1, TMA bytes
  uint64_t* empty = bars + 3;        // [NS] stage consumed: MMA commit, prep warp, epilogue warps
  uint64_t* acc_full = bars + 6;     // [2] accumulators of a unit complete
  uint64_t* acc_empty = bars + 8;    // [2] epilogue done with an accumulator stage
  uint64_t* scal_ready = bars + 10;  // [2] per-position scalars written
  uint64_t* coef_ready = bars + 12;  // Cf of the current unit written (every unit)
  uint64_t* coef_free = bars + 13;   // MMAs of the previous unit done (Cf may be rewritten)
  uint64_t* sready = bars + 14;      // [2] S_ctx buffer loaded into tensor memory
  uint64_t* sfree = bars + 16;       // [2] last MMA reading an S_ctx buffer done
  uint64_t* dec_ready = bars + 18;   // [2] decay table buffer written
  uint64_t* dec_free = bars + 20;    // [2] coefficient warps done with a decay table buffer
  uint64_t* g_ready = bars + 22;     // G of the current unit in tensor memory (units with U > 0)
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 23);
  auto stage = [&](int s) { return smem + size_t(s) * L.stage; };
  auto info = [&](int s) { return reinterpret_cast<MmaInfo*>(stage(s) + L.info_off); };
  unsigned char* CH = smem + L.ch_off;
  unsigned char* CL = smem + L.cl_off;
  float* DEC0 = reinterpret_cast<float*>(smem + L.dec_off);   // [2][32][48]
  MmaScal* SC = reinterpret_cast<MmaScal*>(smem + L.sc_off);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = a.t, n_anc = t - 1;
  // (request, head) pairs dealt round-robin: CTA c takes rh = c, c + G, c + 2G, ... so that at
  // any time the CTAs work on neighbouring heads of the same beams (whose q, k, v, o rows and
  // records lie next to each other in memory)
  int n_my = 0;
  for (int rh = blockIdx.x; rh < a.R * a.H; rh += gridDim.x) n_my += __ldcg(up.ucnt + rh / a.H);

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 32 * kMmaProd + 1);   // cp.async arrivals + header (with bytes)
      mbar_init(&empty[s], 1 + 1 + kMmaEpi);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&acc_full[x], 1);
      mbar_init(&acc_empty[x], kMmaEpi);
      mbar_init(&scal_ready[x], 1);
      mbar_init(&sready[x], kMmaCoef);
      mbar_init(&sfree[x], 1);
      mbar_init(&dec_ready[x], 1);
      mbar_init(&dec_free[x], kMmaCoef);
    }
    mbar_init(coef_ready, kMmaCoef);
    mbar_init(coef_free, 1);
    mbar_init(g_ready, 1);
    fence_barrier_init();
  }
  if (warp == kMmaWMma) tmem_alloc(holder, 512);
  // zero the stages and the Cf tiles once: rows that no unit has filled yet hold finite values
  for (uint32_t x = tid; x < L.dec_off / 16u; x += blockDim.x)
    reinterpret_cast<uint4*>(smem)[x] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  __syncthreads();
  tc_fence_after();
  // tensor memory: columns [128 a, 128 a + 128) accumulator stage a (D1 q | D1 k | D2 q | D2 k),
  // [256 + 128 j, +128) S_ctx buffer j (hi in the first d_k / 2 columns, lo after)
  const uint32_t tmem = *holder;

  if (warp < kMmaProd) {
    // ------------------------------------------------------------------ producers
    const int pw = warp;
    int issued = 0;
    if (n_my > 0) {
      int r = int(blockIdx.x) / a.H, h = int(blockIdx.x) % a.H, k = 0;
      int cnt = __ldcg(up.ucnt + r);
      const int* rec = up.urec + (size_t(r) * up.maxU + k) * kUnitRecInts;
      int x0 = __ldcg(rec + lane), x1 = __ldcg(rec + 32 + lane), x2 = __ldcg(rec + 64 + lane);
      int prev_rh = -1;
      for (int i = 0; i < n_my; ++i) {
        const int s = i % NS, n = i / NS;
        if (i >= NS && !__all_sync(kFull, mbar_wait_bounded(&empty[s], (n - 1) & 1))) {
          if (lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 20, t);
          break;
        }
        // the next unit of the walk; its record is fetched now and used in the next iteration
        int nr = r, nh = h, nk = k + 1, ncnt = cnt;
        if (nk == cnt) {
          nk = 0;
          const int nrh = r * a.H + h + int(gridDim.x);
          nr = nrh / a.H;
          nh = nrh % a.H;
        }
        const bool more = i + 1 < n_my;
        int y0 = 0, y1 = 0, y2 = 0;
        if (more) {
          if (nr != r) ncnt = __ldcg(up.ucnt + nr);
          const int* nrec = up.urec + (size_t(nr) * up.maxU + nk) * kUnitRecInts;
          y0 = __ldcg(nrec + lane);
          y1 = __ldcg(nrec + 32 + lane);
          y2 = __ldcg(nrec + 64 + lane);
        }
        const int rh = r * a.H + h;
        const int first = rh != prev_rh;
        if (first) {
          // S_ctx hi/lo rows of this (request, head) (first unit only) and of the next one,
          // into L2 ahead of the builders' loads: 2 x 128 rows x 2 d_k bytes
          const int nb = (prev_rh < 0 ? 2 : 1);
          for (int q = 0; q < nb; ++q) {
            const int rq = rh + (nb == 2 ? q : 1) * int(gridDim.x);
            if (rq < a.R * a.H) {
              const unsigned char* hi_b = reinterpret_cast<const unsigned char*>(S_hi) + size_t(rq) * DV * DK * 2;
              const unsigned char* lo_b = reinterpret_cast<const unsigned char*>(S_lo) + size_t(rq) * DV * DK * 2;
              for (int x = pw * 32 + lane; x < DV * DK * 2 / 128; x += 32 * kMmaProd) {
                prefetch_l2(hi_b + size_t(x) * 128);
                prefetch_l2(lo_b + size_t(x) * 128);
              }
            }
          }
        }
        const int last = (!more || nr != r || nh != h) ? 1 : 0;
        prev_rh = rh;
        // record: [0] start | n_pos << 16, [1] U, [4 + p] beam, [36 + u] (slot << 16) | beam
        const int sn = __shfl_sync(kFull, x0, 0);
        const int U = min(__shfl_sync(kFull, x0, 1), UC);
        const int start = sn & 0xffff, n_pos = min(sn >> 16, NP);
        const int bA = __shfl_sync(kFull, x0, (lane + 4) & 31);
        const int bB = __shfl_sync(kFull, x1, (lane + 4) & 31);
        const int aB = __shfl_sync(kFull, x2, (lane + 4) & 31);
        const int beam = lane < 28 ? bA : bB;             // position p = lane
        const int anc0 = lane < 28 ? bB : aB;            // record u = lane
        const int anc1 = aB;                             // record u = 32 + lane
        const int io_l = (r * a.B + beam) * a.H + h;
        const int row0 = rec_row_hm(a, anc0 >> 16, r, h, anc0 & 0xffff);
        const int row1 = rec_row_hm(a, anc1 >> 16, r, h, anc1 & 0xffff);
        unsigned char* st = stage(s);
        MmaInfo* inf = info(s);
        // Every operand row goes in by TMA row gathers of four (tile::gather4, 128-byte
        // swizzle, 64 columns per copy), all counted as transaction bytes on full[s]: q, k rows
        // of the position groups, v rows, the ancestor keys and the w records (hi, lo x two
        // halves of d_v). The copies form one list; warp pw issues entries [pw C, pw C + C) in
        // one instruction. Rows past n_pos / U repeat row 0 (never read).
        const int U4 = (U + 3) & ~3, G4 = (n_pos + 3) >> 2;
        const int nqk = 2 * G4 * NSL, nv = 2 * G4, nka = (U4 / 4) * NSL;
        const int nops = nqk + nv + nka + U4;
        if (pw == 0) {
          if (lane == 0) {
            inf->r = r;
            inf->h = h;
            inf->start = start;
            inf->n_pos = n_pos;
            inf->U = U;
            inf->first = first;
            inf->last = last;
          }
          inf->beam[lane] = beam;
          __syncwarp();
          if (lane == 0) mbar_arrive_expect_tx(&full[s], uint32_t(nops) * 512u);
          __syncwarp();
        }
        {
          const int C = (nops + kMmaProd - 1) / kMmaProd;          // <= 20 (<= 120 copies)
          const int id = pw * C + lane;
          const bool has = lane < C && id < nops;
          const int kind = id < nqk ? 0 : id < nqk + nv ? 1 : id < nqk + nv + nka ? 2 : 3;
          int m, xc, sm_off;
          const CUtensorMap* map;
          if (kind == 0) {
            const int side = id / (G4 * NSL), e = id % (G4 * NSL), ks = e % NSL;
            m = e / NSL;
            xc = 64 * ks;
            sm_off = ks * 8192 + (side * NP + 4 * m) * 128;
            map = side ? &mk : &mq;
          } else if (kind == 1) {
            const int e = id - nqk, ks = e & 1;
            m = e >> 1;
            xc = 64 * ks;
            sm_off = int(L.v_off) + ks * (NP * 128) + 4 * m * 128;
            map = &mv;
          } else if (kind == 2) {
            const int e = id - nqk - nv, ks = e % NSL;
            m = e / NSL;
            xc = 64 * ks;
            sm_off = int(L.ka_off) + ks * (UC * 128) + 4 * m * 128;
            map = &mkr;
          } else {
            const int e = id - nqk - nv - nka, pl = (e >> 1) & 1, mb = e & 1;
            m = e >> 2;
            xc = 128 * pl + 64 * mb;
            sm_off = int(pl ? L.wl_off : L.wh_off) + (4 * m >> 3) * 2048 + mb * 1024 + (4 * m & 7) * 128;
            map = &mw;
          }
          int y[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int pj = (4 * m + j) & 63;
            const int yp = __shfl_sync(kFull, io_l, pj < n_pos ? pj : 0);
            const int uu = pj < U ? pj : 0;
            const int rA = __shfl_sync(kFull, row0, uu & 31), rB = __shfl_sync(kFull, row1, uu & 31);
            y[j] = kind <= 1 ? yp : (uu < 32 ? rA : rB);
          }
          if (has) tma_gather4(st + sm_off, map, &full[s], xc, y[0], y[1], y[2], y[3]);
        }
        if (pw == 1) {
          if (lane < n_pos) {
            cp_async4(&inf->gb[2 * lane], a.g + io_l);
            cp_async4(&inf->gb[2 * lane + 1], a.beta + io_l);
            cp_async16(&inf->upos[lane][0], up.upos + (size_t(r) * a.B + start + lane) * 16);
          }
          if (lane < U) cp_async4(&inf->alpha[lane], a.A + row0);
          if (lane + 32 < U) cp_async4(&inf->alpha[32 + lane], a.A + row1);
        }
        cp_async_arrive(&full[s]);
        issued = i + 1;
        x0 = y0;
        x1 = y1;
        x2 = y2;
        r = nr;
        h = nh;
        k = nk;
        cnt = ncnt;
      }
    }
    // the CTA may not exit with copies in flight
    for (int i = issued > NS ? issued - NS : 0; i < issued; ++i)
      mbar_wait_bounded(&full[i % NS], (i / NS) & 1);
  } else if (warp == kMmaWMma) {
    // ------------------------------------------------------------------ MMA (whole warp)
    // The warp runs converged; one elected lane issues each tensor-core instruction.
    // Software-pipelined by one unit: iteration i first finishes unit i - 1 (D2 once its Cf is
    // written, then the commits that hand it to the epilogue), then starts unit i (G, D1). The
    // coefficient warps build Cf of unit i while the tensor pipe runs unit i's D1 and the
    // epilogue drains unit i - 1.
    int sver = -1, last_i = -1;
    int pU = 0, ps = 0, pac = 0, pj = 0, plast = 0;    // the unit whose D2 is pending
    bool ok = true;
    for (int i = 0; i <= n_my && ok; ++i) {
      if (i >= 1) {
        ok = __all_sync(kFull, mbar_wait_bounded(coef_ready, (i - 1) & 1));
        tc_fence_after();
        if (ok) {
          const uint32_t d2 = tmem + uint32_t(pac) * 128u + 64u;
          const uint32_t st = smem_u32(stage(ps));
          const uint32_t id2 = idesc_bf16_f32_amn(128, 2 * NP);
#pragma unroll 1
          for (int kq = 0; kq < (pU + 15) / 16; ++kq) {
            const uint64_t ah = sw128_mnmajor_desc(st + L.wh_off + kq * 4096, 1024, 2048);
            const uint64_t al = sw128_mnmajor_desc(st + L.wl_off + kq * 4096, 1024, 2048);
            const uint64_t bh = sw128_kmajor_desc(smem_u32(CH) + kq * 32);
            const uint64_t bl = sw128_kmajor_desc(smem_u32(CL) + kq * 32);
            umma_bf16_w(d2, ah, bh, id2, kq != 0 ? 1u : 0u);
            umma_bf16_w(d2, al, bh, id2, 1u);
            umma_bf16_w(d2, ah, bl, id2, 1u);
          }
          umma_commit_w(&acc_full[pac]);
          umma_commit_w(coef_free);
          umma_commit_w(&empty[ps]);
          if (plast) umma_commit_w(&sfree[pj]);
          last_i = i - 1;
        }
      }
      if (ok && i < n_my) {
        const int s = i % NS, n = i / NS, ac = i & 1;
        ok = __all_sync(kFull, mbar_wait_bounded(&full[s], n & 1));
        fence_proxy_async_smem();                  // cp.async data -> tensor-core reads
        const MmaInfo* inf = info(s);
        const int U = min(inf->U, UC);
        if (inf->first) ++sver;
        const int j = sver & 1;
        if (i >= 2) ok = ok && __all_sync(kFull, mbar_wait_bounded(&acc_empty[ac], ((i - 2) >> 1) & 1));
        tc_fence_after();
        const uint32_t d1 = tmem + uint32_t(ac) * 128u, d2 = d1 + 64u;
        const uint32_t st = smem_u32(stage(s));
        if (ok && U > 0) {
          // G[x][u] = x . k_u (M = 64 rows x of the q | k tile, N = 48 records), into the
          // columns that D2 overwrites once the coefficient warps have read G
          const uint32_t id0 = idesc_bf16_f32(64, UC);
#pragma unroll 1
          for (int kstep = 0; kstep < DK / 16; ++kstep) {
            const uint32_t ks = uint32_t(kstep >> 2), kk = uint32_t(kstep & 3);
            const uint64_t ax = sw128_kmajor_desc(st + ks * 8192u + kk * 32u);
            const uint64_t bk = sw128_kmajor_desc(st + L.ka_off + ks * (UC * 128u) + kk * 32u);
            umma_bf16_w(d2, ax, bk, id0, kstep != 0 ? 1u : 0u);
          }
          umma_commit_w(g_ready);
        }
        ok = ok && __all_sync(kFull, mbar_wait_bounded(&sready[j], (sver >> 1) & 1));
        tc_fence_after();
        if (ok) {
          const uint32_t sa = tmem + 256u + uint32_t(j) * 128u;
          const uint32_t id1 = idesc_bf16_f32(128, 2 * NP);
#pragma unroll 1
          for (int kstep = 0; kstep < DK / 16; ++kstep) {
            const uint32_t ks = uint32_t(kstep >> 2), kk = uint32_t(kstep & 3);
            const uint64_t bx = sw128_kmajor_desc(st + ks * 8192u + kk * 32u);
            umma_bf16_ts_w(d1, sa + kstep * 8, bx, id1, kstep != 0 ? 1u : 0u);
            umma_bf16_ts_w(d1, sa + DK / 2 + kstep * 8, bx, id1, 1u);
          }
        }
        pU = U;
        ps = s;
        pac = ac;
        pj = j;
        plast = inf->last;
      }
      if (!ok && lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 21, t);
    }
    // tensor memory is released only once the last MMA has completed
    if (last_i >= 0) mbar_wait_bounded(&acc_full[last_i & 1], (last_i >> 1) & 1);
    __syncwarp();
  } else if (warp == kMmaWPrep) {
    // ------------------------------------------------------------------ prep warp
    // Per unit, from the staged data only (nothing here waits for a tensor-core result, so the
    // warp runs ahead): k_p . q_p, the appends of k_p and alpha_p, the decay table and the
    // per-position scalars.
    __nv_bfloat16* kout = static_cast<__nv_bfloat16*>(a.Kr);
    const int gq = lane >> 2, c4 = lane & 3;
    for (int i = 0; i < n_my; ++i) {
      const int s = i % NS, n = i / NS, ac = i & 1;
      bool ok = mbar_wait_bounded(&full[s], n & 1);
      if (i >= 2) {
        ok = ok && mbar_wait_bounded(&acc_empty[ac], ((i - 2) >> 1) & 1);   // SC[ac] free
        ok = ok && mbar_wait_bounded(&dec_free[ac], ((i - 2) >> 1) & 1);    // DEC[ac] free
      }
      if (!__all_sync(kFull, ok)) {
        if (lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 23, t);
        break;
      }
      const MmaInfo* inf = info(s);
      const unsigned char* st = stage(s);
      const int r = inf->r, h = inf->h, n_pos = min(inf->n_pos, NP);
      MmaScal* sc = SC + ac * NP;
      float* DEC = DEC0 + ac * (NP * UC);
      // position p = lane: beam, new record row, decay walk
      const int p = lane;
      const bool valid = p < n_pos;
      const int b = inf->beam[p];
      const int wnew = rec_row_hm(a, t - 1, r, h, b);
      {
        float4* d4 = reinterpret_cast<float4*>(DEC);
        for (int x = lane; x < NP * UC / 4; x += 32) d4[x] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      __syncwarp();
      float e = 0.f, alpha = 0.f, beta = 0.f;
      if (valid) {
        const uint4 ur = *reinterpret_cast<const uint4*>(&inf->upos[p][0]);
        const uint32_t uw[4] = {ur.x, ur.y, ur.z, ur.w};
        int us[kMmaMaxT - 1];
        float al[kMmaMaxT - 1];
#pragma unroll
        for (int sl = 0; sl < kMmaMaxT - 1; ++sl) {
          us[sl] = min(int((uw[sl >> 2] >> (8 * (sl & 3))) & 0xffu), UC - 1);
          al[sl] = sl < n_anc ? inf->alpha[us[sl]] : 1.f;
        }
        float x = 1.f;
#pragma unroll
        for (int sl = kMmaMaxT - 2; sl >= 0; --sl) {
          if (sl < n_anc) {
            DEC[p * UC + us[sl]] = x;
            x *= al[sl];
          }
        }
        e = x;
        alpha = expf(inf->gb[2 * p]);
        beta = inf->gb[2 * p + 1];
        a.A[wnew] = alpha;
      }
      sc[p].e = e;
      sc[p].alpha = alpha;
      sc[p].beta = beta;
      sc[p].io = (r * a.B + b) * a.H + h;
      sc[p].wnew = wnew;
      sc[p].valid = valid ? 1 : 0;
      // k_p . q_p: the diagonal of Xq Xk^T on warp-level MMA, 16 x 8 tiles along the diagonal
      {
        const uint32_t xb = smem_u32(st);
        float acc[2][2][4];
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) acc[m][hh][0] = acc[m][hh][1] = acc[m][hh][2] = acc[m][hh][3] = 0.f;
#pragma unroll 2
        for (int kq = 0; kq < DK / 16; ++kq) {
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const int an = 16 * m + (lane & 15), kc = 2 * kq + (lane >> 4);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(xb + (kc >> 3) * 8192 + an * 128 + (((kc & 7) ^ (an & 7)) << 4), a0, a1, a2, a3);
            const int bn = 32 + 16 * m + 8 * (lane >> 4) + (lane & 7), bc = 2 * kq + ((lane >> 3) & 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(xb + (bc >> 3) * 8192 + bn * 128 + (((bc & 7) ^ (bn & 7)) << 4), b0, b1, b2, b3);
            mma_16816_bf16(acc[m][0], a0, a1, a2, a3, b0, b1);
            mma_16816_bf16(acc[m][1], a0, a1, a2, a3, b2, b3);
          }
        }
        // lane (g, c) with c = g / 2 holds the diagonal entries of rows g and g + 8 of a tile
        if (c4 == (gq >> 1)) {
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            sc[16 * m + gq].c0 = (gq & 1) ? acc[m][0][1] : acc[m][0][0];
            sc[16 * m + 8 + gq].c0 = (gq & 1) ? acc[m][1][3] : acc[m][1][2];
          }
        }
      }
      // append k_p (two rows of 256 bytes per warp instruction)
      {
        constexpr int RPI = 32 / CR;
        const int c = lane % CR;
#pragma unroll 4
        for (int j = 0; j < NP / RPI; ++j) {
          const int pp = j * RPI + lane / CR, nn = 32 + pp;
          const int wr = __shfl_sync(kFull, wnew, pp);
          if (pp < n_pos) {
            const uint4 v = *reinterpret_cast<const uint4*>(
                st + (c >> 3) * 8192 + nn * 128 + (((c & 7) ^ (nn & 7)) << 4));
            *reinterpret_cast<uint4*>(kout + size_t(wr) * DK + c * 8) = v;
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&dec_ready[ac]);
        mbar_arrive(&scal_ready[ac]);
        mbar_arrive(&empty[s]);
      }
    }
  } else if (warp < kMmaWEpi) {
    // ------------------------------------------------------------------ coefficient warps
    const int sp = warp & 3;
    int sver = -1, gcnt = 0;
    for (int i = 0; i < n_my; ++i) {
      const int s = i % NS, n = i / NS, ac = i & 1;
      bool ok = mbar_wait_bounded(&full[s], n & 1);
      const MmaInfo* inf = info(s);
      const int r = inf->r, h = inf->h, U = min(inf->U, UC);
      if (inf->first) {
        ++sver;
        const int j = sver & 1;
        if (sver >= 2) ok = ok && mbar_wait_bounded(&sfree[j], ((sver >> 1) - 1) & 1);
        if (!__all_sync(kFull, ok)) {
          if (lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 22, t);
          break;
        }
        // S_ctx rows 32 sp .. 32 sp + 31 (hi, then lo) into buffer j; one row per lane, two bf16
        // per 32-bit column, lower k in the low half (memory order); four 16-byte loads per
        // tensor-memory store (the rows were prefetched into L2 by the producers)
        tc_fence_after();
        const int row = 32 * sp + lane;
        const size_t rh = size_t(r) * a.H + h;
        const uint32_t ta = tmem + (uint32_t(32 * sp) << 16) + 256u + uint32_t(j) * 128u;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint4* src = reinterpret_cast<const uint4*>((half ? S_lo : S_hi) +
                                                            (rh * DV + row) * DK);
#pragma unroll 1
          for (int c4 = 0; c4 < DK / 32; ++c4) {
            const uint4 w4[4] = {__ldg(src + 4 * c4), __ldg(src + 4 * c4 + 1), __ldg(src + 4 * c4 + 2),
                                 __ldg(src + 4 * c4 + 3)};
            tmem_st16(ta + half * (DK / 2) + c4 * 16, w4);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sready[j]);
      }
      // the decay table (always waited, so these warps never run two units ahead of the prep
      // warp), G, and the previous unit's MMAs (waited at every unit so that the wait never
      // falls two phases behind the barrier)
      ok = ok && mbar_wait_bounded(&dec_ready[ac], (i >> 1) & 1);
      if (U > 0) {
        ok = ok && mbar_wait_bounded(g_ready, gcnt & 1);
        ++gcnt;
      }
      if (i >= 1) ok = ok && mbar_wait_bounded(coef_free, (i - 1) & 1);
      if (!__all_sync(kFull, ok)) {
        if (lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 25, t);
        break;
      }
      tc_fence_after();
      if (U > 0) {
        // Cf = DEC * G, written as bf16 hi + lo, 16 records at a time. Thread n = 16 sp + lane
        // (lanes 0-15) holds row n of G (the M = 64 layout puts rows 16 sp .. 16 sp + 15 in
        // lanes 0-15 of subpartition sp).
        const uint32_t tg = tmem + (uint32_t(32 * sp) << 16) + uint32_t(ac) * 128u + 64u;
        const int nrow = 16 * sp + (lane & 15), p = nrow & 31;
        const float* dr = DEC0 + ac * (NP * UC) + p * UC;
#pragma unroll 1
        for (int h16 = 0; h16 < UC / 16; ++h16) {
          if (16 * h16 >= U) break;                   // warp-uniform
          float gr[16];
          tmem_ld16(tg + 16u * h16, gr);
          if (lane < 16) {
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
              const int q = 2 * h16 + q2;
              const float4 d0 = *reinterpret_cast<const float4*>(dr + 8 * q);
              const float4 d1 = *reinterpret_cast<const float4*>(dr + 8 * q + 4);
              const float v[8] = {gr[8 * q2] * d0.x,     gr[8 * q2 + 1] * d0.y,
                                  gr[8 * q2 + 2] * d0.z, gr[8 * q2 + 3] * d0.w,
                                  gr[8 * q2 + 4] * d1.x, gr[8 * q2 + 5] * d1.y,
                                  gr[8 * q2 + 6] * d1.z, gr[8 * q2 + 7] * d1.w};
              uint32_t hw[4], lw[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 hi2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
                const float2 hf2 = __bfloat1622float2(hi2);
                const __nv_bfloat162 lo2 =
                    __floats2bfloat162_rn(v[2 * e] - hf2.x, v[2 * e + 1] - hf2.y);
                hw[e] = *reinterpret_cast<const uint32_t*>(&hi2);
                lw[e] = *reinterpret_cast<const uint32_t*>(&lo2);
              }
              const uint32_t off = uint32_t(nrow) * 128u + uint32_t((q ^ (nrow & 7)) << 4);
              *reinterpret_cast<uint4*>(CH + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              *reinterpret_cast<uint4*>(CL + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
          }
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&dec_free[ac]);
        mbar_arrive(coef_ready);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    // thread = state row (tensor-memory lane); warp (sp, ph) = rows 32 sp.., positions 16 ph..
    const int ew = warp - kMmaWEpi, sp = warp & 3, ph = ew >> 2;
    const int row = 32 * sp + lane;
    const uint32_t tl = tmem + (uint32_t(32 * sp) << 16);
    __nv_bfloat16* Wb = reinterpret_cast<__nv_bfloat16*>(a.W);
    for (int i = 0; i < n_my; ++i) {
      const int s = i % NS, ac = i & 1;
      bool ok = mbar_wait_bounded(&acc_full[ac], (i >> 1) & 1);
      ok = ok && mbar_wait_bounded(&scal_ready[ac], (i >> 1) & 1);
      if (!__all_sync(kFull, ok)) {
        if (lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 26, t);
        break;
      }
      tc_fence_after();
      const MmaScal* sc = SC + ac * NP;
      const unsigned char* Vb = stage(s) + L.v_off;   // [2][32][128 B] sw128
      const MmaInfo* inf = info(s);
      const int n_pos = min(inf->n_pos, NP), U = inf->U;
      const uint32_t base = tl + uint32_t(ac) * 128u;
#pragma unroll 1
      for (int pb = 0; pb < 2; ++pb) {
        const int p0 = 16 * ph + 8 * pb;
        if (p0 < n_pos) {                             // warp-uniform
          float q1[8], k1[8], q2[8], k2[8];
          tmem_ld8x4(base + p0, base + NP + p0, base + 2 * NP + p0, base + 3 * NP + p0, q1, k1,
                     q2, k2);
          if (U == 0) {
#pragma unroll
            for (int j = 0; j < 8; ++j) q2[j] = k2[j] = 0.f;
          }
          // four positions at a time: their scalars and v first, then the stores (loads issued
          // ahead of the stores, which the compiler cannot move them past)
#pragma unroll
          for (int j4 = 0; j4 < 8; j4 += 4) {
            float4 sa[4];
            int io[4], wn[4];
            float vv[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const int pp = p0 + j4 + jj;
              sa[jj] = *reinterpret_cast<const float4*>(&sc[pp]);
              const int4 sb = *reinterpret_cast<const int4*>(&sc[pp].io);
              io[jj] = sb.x;
              wn[jj] = sb.y;
              vv[jj] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                  Vb + (row >> 6) * (NP * 128) + pp * 128 + ((((row & 63) >> 3) ^ (pp & 7)) << 4) +
                  (row & 7) * 2));
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const int j = j4 + jj;
              if (p0 + j < n_pos) {
                const float uu = fmaf(sa[jj].x, k1[j], k2[j]);
                const float qq = fmaf(sa[jj].x, q1[j], q2[j]);
                const float w = sa[jj].z * (vv[jj] - sa[jj].y * uu);
                const float o = fmaf(sa[jj].y, qq, sa[jj].w * w);
                a.o[size_t(io[jj]) * DV + row] = o;
                const __nv_bfloat16 whi = __float2bfloat16_rn(w);
                const __nv_bfloat16 wlo = __float2bfloat16_rn(w - __bfloat162float(whi));
                Wb[size_t(wn[jj]) * (2 * DV) + row] = whi;
                Wb[size_t(wn[jj]) * (2 * DV) + DV + row] = wlo;
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&acc_empty[ac]);
        mbar_arrive(&empty[s]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------- host side

bool replay_mma_supported(int d_k, int d_v, int B, int T_max) {
  return d_v == kMmaDV && (d_k == 64 || d_k == 128) && T_max <= kMmaMaxT && B <= kMmaMaxB;
}

size_t replay_mma_smem(int d_k) { return mma_layout(d_k).bytes; }

cudaError_t launch_plan_units(const StepArgs& a, const UnitPlan& up, cudaStream_t stream);

bool make_rows_map(CUtensorMap* map, const void* base, uint64_t rows, int cols,
                   uint64_t row_bytes);

// Tensor maps of the key and w records (fixed for a handle): Kr [T_max R H B][d_k] bf16 and
// W [T_max R H B][2 d_v] bf16 (hi plane, lo plane).
bool make_record_maps(CUtensorMap* mkr, CUtensorMap* mw, const void* Kr, const void* W,
                      uint64_t n_rec, int d_k, int d_v) {
  return make_rows_map(mkr, Kr, n_rec, d_k, uint64_t(d_k) * 2) &&
         make_rows_map(mw, W, n_rec, 2 * d_v, uint64_t(d_v) * 4);
}

template <int DK>
static cudaError_t launch_mma_t(const void* S_hi, const void* S_lo, const StepArgs& a,
                                const UnitPlan& up, const CUtensorMap& mq, const CUtensorMap& mk,
                                const CUtensorMap& mv, const CUtensorMap& mkr, const CUtensorMap& mw,
                                int n_sm,
                                cudaStream_t stream) {
  const MmaLayout L = mma_layout(DK);
  auto kern = replay_mma_kernel<DK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(L.bytes));
  if (e != cudaSuccess) return e;
  kern<<<n_sm, kMmaWarps * 32, L.bytes, stream>>>(static_cast<const __nv_bfloat16*>(S_hi),
                                                  static_cast<const __nv_bfloat16*>(S_lo), a, up,
                                                  mq, mk, mv, mkr, mw);
  return cudaGetLastError();
}

// S_hi, S_lo: the shared state split into bf16 hi + lo, [R*H][128][d_k]. W records are stored
// as [hi plane | lo plane] bf16 rows of 2 d_v elements. mkr, mw from make_record_maps; the
// q, k and v maps are made here for this step's inputs.
cudaError_t launch_replay_mma(const StepArgs& a, const UnitPlan& up, const void* S_hi,
                              const void* S_lo, const CUtensorMap& mkr, const CUtensorMap& mw,
                              cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  const uint64_t rows = uint64_t(a.R) * a.B * a.H;
  if (!make_rows_map(&mq, a.q, rows, a.d_k, uint64_t(a.d_k) * 2) ||
      !make_rows_map(&mk, a.k, rows, a.d_k, uint64_t(a.d_k) * 2) ||
      !make_rows_map(&mv, a.v, rows, kMmaDV, uint64_t(kMmaDV) * 2))
    return cudaErrorInvalidValue;
  cudaError_t e = launch_plan_units(a, up, stream);
  if (e != cudaSuccess) return e;
  int dev = 0, n_sm = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (a.d_k == 64) return launch_mma_t<64>(S_hi, S_lo, a, up, mq, mk, mv, mkr, mw, n_sm, stream);
  if (a.d_k == 128) return launch_mma_t<128>(S_hi, S_lo, a, up, mq, mk, mv, mkr, mw, n_sm, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ola
