// Projection-replay decode step with both contractions on tensor cores: persistent, pipelined,
// state-major (sm_100a; d_k, d_v in {64, 128, 256}, T_max <= 12, B <= 1024, bf16 inputs).
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
// Rows of the state never mix: u_p[i], w_p[i] and o_p[i] use row i of S_ctx and of the w
// records only, while G and Cf depend on the keys alone. A state of d_v = 256 rows is therefore
// decoded as two independent blocks of 128 rows (each a (request, head, row block) walk item with
// its own S_ctx rows in tensor memory; G is formed in both). At d_v = 64 the M = 128 tensor-core
// rows hold the state twice (S_ctx rows 0..63 again in tensor-memory lanes 64..127, and the w
// planes' second 64-row block read from the first one): D1 and D2 then carry every position in
// both halves, and the epilogue warps of lanes 0..63 finish positions 0..15 while those of lanes
// 64..127 finish positions 16..31, so all eight epilogue warps share the unit.
//
// One CTA per SM walks the units of its (request, head, row block) items, dealt round-robin,
// through an operand ring (three stages, two at d_k = 256) and a ring of v rows and unit
// headers (four slots, three at d_k = 256). Warp roles:
//   warps 0-2, 4-5  producers: TMA row gathers (tile::gather4, 128-byte swizzle) of the unit's
//               q, k and v rows, distinct ancestor keys and w records (the latter as the
//               MN-major operand), one list of copies dealt out in five chunks; cp.async of
//               the per-position scalars.
//   warp 3      head MMA: G with the staged q, k tile as A and the ancestor keys as B; D1 with
//               S_ctx (bf16 hi + lo) held in tensor memory as the A operand. Three accumulator
//               stages (two at d_k = 256, where S_ctx takes 256 tensor-memory columns).
//   warp 6      tail MMA: D2 with the staged w planes as the A operand and Cf as B, written
//               over G.
//   warp 7      prep: decay table, per-position scalars, append of alpha_p (row block 0).
//   warps 8-11  coefficients: S_ctx into tensor memory when the walk item changes;
//               k_p . q_p and the append of k_p (row block 0); Cf from G and the decay table.
//   warps 12-19 epilogue: thread = state row i; w_p[i] and o_p[i] from D1, D2 and the scalars;
//               stores o (fp32) and the w record (hi, lo).
// Every wait is bounded; on timeout the kernel records OLA_ERR_TIMEOUT and finishes.
#include "ola_device.cuh"

namespace ola {

constexpr int kMmaMaxT = 12;
constexpr int kMmaMaxB = 1024;

// Pipeline depths, unit size and row blocking for a geometry. Tensor memory: NA accumulator
// stages of 128 columns, then S_ctx hi | lo (DK columns); shared memory: NS operand stages of
// which the ancestor keys and w planes are sized for UC records, and NB v slots. A unit holds at
// most UC distinct ancestor records (the plan cuts units to that).
template <int DK, int DV>
struct MmaCfg {
  static constexpr int NRB = DV > 128 ? DV / 128 : 1;   // 128-row blocks of the state
  static constexpr int DVB = DV < 128 ? DV : 128;       // state rows of one block
  static constexpr int NVH = DVB / 64;                  // 64-column halves of a block's v row
  static constexpr int UC = kUnitAnc;
  static constexpr int NS = DK > 128 ? 2 : 3;
  static constexpr int NB = DK > 128 ? 3 : 4;
  static constexpr int NA = DK > 128 ? 2 : 3;
  static_assert(128 * NA + DK <= 512, "tensor memory: accumulators and S_ctx");
  static_assert(UC % 16 == 0 && UC <= kUnitAnc, "records come in MMA K-steps of 16");
};
// A TMA instruction holds its warp for several hundred cycles plus roughly eighty per active
// lane, while the instructions of different warps proceed in parallel: the copies of a unit are
// spread over five producer warps, one warp-wide gather instruction each.
// Two warps issue tensor-core work: the head warp (G and D1 of a unit, as soon as its operands
// and an accumulator stage are there) and the tail warp (D2 once Cf is written), so that the
// tensor pipe is fed from both ends of the pipeline.
// Warp w runs on subpartition w % 4. Every subpartition holds one coefficient warp and two
// epilogue warps (their tensor-memory lane quarter is w % 4).
constexpr int kMmaProd = 5, kMmaCoef = 4, kMmaEpi = 8;
constexpr int kMmaWarps = kMmaProd + 3 + kMmaCoef + kMmaEpi;   // 20 warps, 5 per subpartition
constexpr int kMmaWMma = 3;                     // head MMA warp
constexpr int kMmaWTail = 6;                    // tail MMA warp
constexpr int kMmaWPrep = 7;
constexpr int kMmaWCoef = 8;                    // warps 8..11 (subpartitions 0..3)
constexpr int kMmaWEpi = kMmaWCoef + kMmaCoef;  // warps 12..19
static_assert(kMmaWCoef % 4 == 0 && kMmaWEpi % 4 == 0, "tensor-memory lane quarters follow warp % 4");
static_assert(kMmaWCoef == kMmaProd + 3, "warps 0..7 are the producers, the MMA and the prep warps");

// Record row of (step slot, request r, beam b, head h) in this kernel's record storage, which
// keeps the heads of a beam next to each other: [T_max][R][B][H] (the heads of one beam are
// decoded at about the same time by neighbouring CTAs, so their rows share DRAM pages).
__device__ __forceinline__ int rec_row_hm(const StepArgs& a, int slot, int r, int h, int b) {
  return ((slot * a.R + r) * a.B + b) * a.H + h;
}

struct MmaInfo {                 // per stage
  int r, h, start, n_pos;
  int U, first, last, rb;        // rb: row block of the walk item
  int beam[kUnitPos];
  float gb[2 * kUnitPos];        // (g, beta) of each position
  float alpha[kUnitAnc];         // alpha of each distinct record
  uint8_t upos[kUnitPos][16];    // record index u of each (position, chain slot)
};

struct MmaScal {                 // per position
  float e, alpha, beta, c0;
  int io, wnew, valid, pad;
};

// Shared memory (every tile 1024-byte aligned). The operand stages are released once the
// unit's MMAs and the coefficient warps are done with them; the v slots and unit headers, read
// by the epilogue, live in a deeper ring of their own.
//   operand stage s < NS: X [NSL][64 rows: q of positions 0-31 | k of positions 0-31][128 B]
//                           K-major, sw128
//                         KA [NSL][48 rows][128 B]   ancestor keys, same swizzle
//                         WH, WL [6 groups of 8 records][2 halves of the row block][8][128 B]
//                           MN-major (at d_v = 64 the second half stays zero)
//   v slot b < NB: V [NVH halves of the row block][32 positions][128 B]  sw128
//   MmaInfo [NB], then CH, CL [64 rows][128 B] (Cf hi, lo; K-major, sw128), DEC [2][32][48]
//   fp32, SC [NB][32] (per-position scalars, by v slot), barriers.
struct MmaLayout {
  uint32_t ka_off, wh_off, wl_off, stage, v_off, info_off;
  uint32_t ch_off, cl_off, dec_off, sc_off, bar_off, bytes;
};

__host__ __device__ inline MmaLayout mma_layout(int d_k, int nvh, int ns, int nb, int na,
                                                int uc) {
  const uint32_t NSL = uint32_t(d_k) / 64u;
  MmaLayout L;
  L.ka_off = NSL * 8192u;
  L.wh_off = L.ka_off + NSL * uint32_t(uc) * 128u;
  L.wl_off = L.wh_off + uint32_t(uc / 8) * 2048u;
  L.stage = L.wl_off + uint32_t(uc / 8) * 2048u;
  L.v_off = uint32_t(ns) * L.stage;
  L.info_off = L.v_off + uint32_t(nb * nvh) * kUnitPos * 128u;
  L.ch_off = (L.info_off + uint32_t(nb) * uint32_t(sizeof(MmaInfo)) + 1023u) & ~1023u;
  L.cl_off = L.ch_off + 8192u;
  L.dec_off = L.cl_off + 8192u;
  L.sc_off = L.dec_off + 2u * kUnitPos * uint32_t(uc) * 4u;
  L.bar_off = L.sc_off + uint32_t(nb) * kUnitPos * uint32_t(sizeof(MmaScal));
  L.bytes = L.bar_off + 320u + 1024u;
  return L;
}

template <int DK, int DV>
__host__ __device__ inline MmaLayout mma_layout_of() {
  using C = MmaCfg<DK, DV>;
  return mma_layout(DK, C::NVH, C::NS, C::NB, C::NA, C::UC);
}

template <int DK, int DV>
__global__ void __launch_bounds__(kMmaWarps * 32, 1)
replay_mma_kernel(const __nv_bfloat16* __restrict__ S_hi, const __nv_bfloat16* __restrict__ S_lo,
                  StepArgs a, UnitPlan up, const __grid_constant__ CUtensorMap mq,
                  const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                  const __grid_constant__ CUtensorMap mkr, const __grid_constant__ CUtensorMap mw) {
  using Cfg = MmaCfg<DK, DV>;
  constexpr int NS = Cfg::NS, NB = Cfg::NB, NA = Cfg::NA, UC = Cfg::UC, NP = kUnitPos;
  constexpr int NRB = Cfg::NRB, DVB = Cfg::DVB, NVH = Cfg::NVH;
  constexpr int MP = NRB * 128;    // rows of S_hi / S_lo per (request, head)
  constexpr int CR = DK / 8;       // 16-byte chunks of a key row
  constexpr int NSL = DK / 64;     // 64-column slices of a key row
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align_smem_1024(smem_raw);
  const MmaLayout L = mma_layout_of<DK, DV>();
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* fullA = bars;              // [NS] operand stage loaded: header arrive + TMA bytes
  uint64_t* emptyA = fullA + NS;       // [NS] operand stage consumed: 2 MMA commits, coef warps
  uint64_t* fullB = emptyA + NS;       // [NB] v slot and header loaded: cp.async arrivals + 1, bytes
  uint64_t* emptyB = fullB + NB;       // [NB] v slot consumed: epilogue warps
  uint64_t* acc_full = emptyB + NB;    // [NA] accumulators of a unit complete (D1 and D2 commits)
  uint64_t* acc_empty = acc_full + NA; // [NA] epilogue done with an accumulator stage
  uint64_t* scal_ready = acc_empty + NA;  // [NB] per-position scalars written (by v slot)
  uint64_t* g_ready = scal_ready + NB;    // [NA] G of a unit in tensor memory (every unit)
  uint64_t* dec_ready = g_ready + NA;     // [2] decay table buffer written
  uint64_t* dec_free = dec_ready + 2;     // [2] coefficient warps done with a decay table buffer
  uint64_t* coef_ready = dec_free + 2;    // Cf of the current unit written (every unit)
  uint64_t* coef_free = coef_ready + 1;   // D2 of the previous unit done (Cf may be rewritten)
  uint64_t* sready = coef_free + 1;    // S_ctx loaded into tensor memory
  uint64_t* sfree = sready + 1;        // last MMA reading S_ctx done
  uint32_t* holder = reinterpret_cast<uint32_t*>(sfree + 1);
  static_assert((2 * NS + 3 * NB + 3 * NA + 8) * 8 + 8 <= 320, "barrier area");
  auto stage = [&](int s) { return smem + size_t(s) * L.stage; };
  auto vslot = [&](int b) { return smem + L.v_off + size_t(b) * (NP * NVH * 128); };
  auto info = [&](int b) { return reinterpret_cast<MmaInfo*>(smem + L.info_off) + b; };
  unsigned char* CH = smem + L.ch_off;
  unsigned char* CL = smem + L.cl_off;
  float* DEC0 = reinterpret_cast<float*>(smem + L.dec_off);   // [2][32][48]
  MmaScal* SC = reinterpret_cast<MmaScal*>(smem + L.sc_off);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = a.t, n_anc = t - 1;
  // Walk items (request, head, row block), row block fastest, dealt round-robin: CTA c takes
  // items c, c + G, c + 2G, ... so that at any time the CTAs work on the row blocks and
  // neighbouring heads of the same beams (whose q, k, v, o rows and records lie next to each
  // other in memory, and whose q / k rows a second row block finds in L2). When items hold many
  // units (4 or more on average), only the full rounds of G items are dealt that way: the units
  // of the remaining items (the tail, items T0 .. n_items - 1, units in item order) are split
  // into G contiguous ranges, one per CTA, so that the last round does not leave CTAs idle.
  // Units in item order: item it of request r starts at unit H NRB uoff[r] + (it - r H NRB)
  // ucnt[r].
  const int HN = a.H * NRB;
  const int n_items = a.R * HN;
  const int GX = int(gridDim.x);
  const bool split_tail = HN * __ldcg(up.uoff + a.R) >= 4 * n_items;
  const int F = split_tail ? n_items / GX : (n_items + GX - 1) / GX;   // rounds dealt round-robin
  const int T0 = split_tail ? F * GX : n_items;                         // first item of the tail
  int tail_begin = 0, n_tail = 0;
  if (T0 < n_items) {
    const int r0 = T0 / HN;
    const int U0 = HN * __ldcg(up.uoff + r0) + (T0 - r0 * HN) * __ldcg(up.ucnt + r0);
    const int NT = HN * __ldcg(up.uoff + a.R) - U0;
    tail_begin = U0 + int((long long)NT * blockIdx.x / GX);
    n_tail = U0 + int((long long)NT * (blockIdx.x + 1) / GX) - tail_begin;
  }
  int n_my = n_tail;
  for (int f = 0; f < F; ++f) {
    const int it = int(blockIdx.x) + f * GX;
    if (it < T0) n_my += __ldcg(up.ucnt + it / HN);
  }

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&fullA[s], 1);                  // expect-tx arrival (with the bytes)
      mbar_init(&emptyA[s], 2 + kMmaCoef);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&fullB[b], 32 * kMmaProd + 1);  // cp.async arrivals + header (with bytes)
      mbar_init(&emptyB[b], kMmaEpi);
      mbar_init(&scal_ready[b], 1 + kMmaCoef);   // prep warp, c0 from the coefficient warps
    }
    for (int x = 0; x < NA; ++x) {
      mbar_init(&acc_full[x], 2);
      mbar_init(&g_ready[x], 1);
      mbar_init(&acc_empty[x], kMmaEpi);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&dec_ready[x], 1);
      mbar_init(&dec_free[x], kMmaCoef);
    }
    mbar_init(coef_ready, kMmaCoef);
    mbar_init(coef_free, 1);
    mbar_init(sready, kMmaCoef);
    mbar_init(sfree, 1);
    fence_barrier_init();
  }
  if (warp == kMmaWMma) tmem_alloc(holder, 512);
  // zero the stages, v slots and Cf tiles once: rows no unit has filled yet hold finite values
  for (uint32_t x = tid; x < L.dec_off / 16u; x += blockDim.x)
    reinterpret_cast<uint4*>(smem)[x] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  __syncthreads();
  tc_fence_after();
  // tensor memory: columns [128 a, 128 a + 128) accumulator stage a < 3 (D1 q | D1 k | D2 q |
  // D2 k), [384, 512) S_ctx (hi in the first d_k / 2 columns, lo after)
  const uint32_t tmem = *holder;

  if (warp < kMmaWCoef && warp != kMmaWMma && warp != kMmaWTail && warp != kMmaWPrep) {
    // ------------------------------------------------------------------ producers
    const int pw = warp < kMmaWMma ? warp : warp - 1;     // 0..4
    int issued = 0;
    // the item and unit holding global unit index u (item-major order)
    auto locate = [&](int u, int& it_, int& r_, int& k_) {
      int lo = 0, hi = a.R - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (HN * __ldcg(up.uoff + mid) <= u) lo = mid;
        else hi = mid - 1;
      }
      r_ = lo;
      const int c_ = __ldcg(up.ucnt + lo);
      const int rem = u - HN * __ldcg(up.uoff + lo);
      it_ = lo * HN + rem / c_;
      k_ = rem % c_;
    };
    if (n_my > 0) {
      int it = int(blockIdx.x), k = 0, r = 0;
      bool tail = F == 0;
      if (tail) locate(tail_begin, it, r, k);
      r = it / HN;
      int h = (it / NRB) % a.H, rb = it % NRB;
      int cnt = __ldcg(up.ucnt + r);
      const int* rec = up.urec + (size_t(r) * up.maxU + k) * kUnitRecInts;
      int x0 = __ldcg(rec + lane), x1 = __ldcg(rec + 32 + lane), x2 = __ldcg(rec + 64 + lane);
      int prev_it = -1;
      for (int i = 0; i < n_my; ++i) {
        const int s = i % NS, n = i / NS, sb = i % NB, nb = i / NB;
        bool okw = i < NS || mbar_wait_bounded(&emptyA[s], (n - 1) & 1);
        if (i >= NB) okw = okw && mbar_wait_bounded(&emptyB[sb], (nb - 1) & 1);
        if (!__all_sync(kFull, okw)) {
          if (lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 20, t);
          break;
        }
        // the next unit of the walk; its record is fetched now and used in the next iteration
        int nit = it, nr = r, nh = h, nrb = rb, nk = k + 1, ncnt = cnt;
        bool ntail = tail;
        if (nk == cnt) {
          nk = 0;
          if (tail) {
            nit = it + 1;
          } else {
            nit = it + GX;
            if (nit >= T0 && n_tail > 0) {
              int rr;
              locate(tail_begin, nit, rr, nk);
              ntail = true;
            }
          }
          nr = nit / HN;
          nh = (nit / NRB) % a.H;
          nrb = nit % NRB;
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
        const int first = it != prev_it;
        if (first) {
          // S_ctx hi/lo rows of this walk item (first unit only) and of the next one, into L2
          // ahead of the coefficient warps' loads: 2 x DVB rows x 2 d_k bytes
          const int npf = (prev_it < 0 ? 2 : 1);
          for (int q = 0; q < npf; ++q) {
            const int iq = (tail || it + GX >= T0) ? it + (npf == 2 ? q : 1) : it + (npf == 2 ? q : 1) * GX;
            if (iq < n_items) {
              const size_t row0 = size_t(iq / NRB) * MP + size_t(iq % NRB) * 128;
              const unsigned char* hi_b = reinterpret_cast<const unsigned char*>(S_hi + row0 * DK);
              const unsigned char* lo_b = reinterpret_cast<const unsigned char*>(S_lo + row0 * DK);
              for (int x = pw * 32 + lane; x < DVB * DK * 2 / 128; x += 32 * kMmaProd) {
                prefetch_l2(hi_b + size_t(x) * 128);
                prefetch_l2(lo_b + size_t(x) * 128);
              }
            }
          }
        }
        const int last = (!more || nit != it) ? 1 : 0;
        prev_it = it;
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
        unsigned char* vs = vslot(sb);
        MmaInfo* inf = info(sb);
        // Every operand row goes in by TMA row gathers of four (tile::gather4, 128-byte
        // swizzle, 64 columns per copy): q, k rows of the position groups, the ancestor keys
        // and the w records (hi, lo x two halves of d_v) into the operand stage, counted as
        // transaction bytes on fullA[s]; the v rows into the v slot, counted on fullB[sb]. The
        // copies form one list; warp pw issues entries [pw C, pw C + C) in one instruction.
        // Rows past n_pos / U repeat row 0 (never read).
        // copies: q / k rows (two sides x G4 groups x NSL slices), v rows (G4 groups x NVH
        // halves), ancestor keys (U4 / 4 groups x NSL slices), w records (U4 / 4 groups x hi, lo
        // x NVH halves)
        const int U4 = (U + 3) & ~3, G4 = (n_pos + 3) >> 2;
        const int nqk = 2 * G4 * NSL, nv = NVH * G4, nka = (U4 / 4) * NSL;
        const int nops = nqk + nv + nka + (U4 / 4) * 2 * NVH;
        if (pw == 0) {
          if (lane == 0) {
            inf->r = r;
            inf->h = h;
            inf->start = start;
            inf->n_pos = n_pos;
            inf->U = U;
            inf->first = first;
            inf->last = last;
            inf->rb = rb;
          }
          inf->beam[lane] = beam;
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_expect_tx(&fullA[s], uint32_t(nops - nv) * 512u);
            mbar_arrive_expect_tx(&fullB[sb], uint32_t(nv) * 512u);
          }
          __syncwarp();
        }
        // warp pw issues entries [pw C, pw C + C), one per lane, 32 at a time (C <= 36: at most
        // 176 copies at d_k = 256, d_v >= 128)
        const int C = (nops + kMmaProd - 1) / kMmaProd;
#pragma unroll 1
        for (int c0 = 0; c0 < C; c0 += 32) {
          const int id = pw * C + c0 + lane;
          const bool has = c0 + lane < C && id < nops;
          const int kind = id < nqk ? 0 : id < nqk + nv ? 1 : id < nqk + nv + nka ? 2 : 3;
          int m, xc;
          unsigned char* dst;
          uint64_t* bar = &fullA[s];
          const CUtensorMap* map;
          if (kind == 0) {
            const int side = id >= G4 * NSL ? 1 : 0, e = id - side * G4 * NSL, ks = e % NSL;
            m = e / NSL;
            xc = 64 * ks;
            dst = st + ks * 8192 + (side * NP + 4 * m) * 128;
            map = side ? &mk : &mq;
          } else if (kind == 1) {
            const int e = id - nqk, ks = e % NVH;
            m = e / NVH;
            xc = rb * 128 + 64 * ks;
            dst = vs + ks * (NP * 128) + 4 * m * 128;
            bar = &fullB[sb];
            map = &mv;
          } else if (kind == 2) {
            const int e = id - nqk - nv, ks = e % NSL;
            m = e / NSL;
            xc = 64 * ks;
            dst = st + L.ka_off + ks * (UC * 128) + 4 * m * 128;
            map = &mkr;
          } else {
            const int e = id - nqk - nv - nka, mb = e % NVH, pl = (e / NVH) & 1;
            m = e / (2 * NVH);
            xc = DV * pl + rb * 128 + 64 * mb;
            dst = st + (pl ? L.wl_off : L.wh_off) + (4 * m >> 3) * 2048 + mb * 1024 + (4 * m & 7) * 128;
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
          if (has) tma_gather4(dst, map, bar, xc, y[0], y[1], y[2], y[3]);
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
        cp_async_arrive(&fullB[sb]);
        issued = i + 1;
        x0 = y0;
        x1 = y1;
        x2 = y2;
        it = nit;
        tail = ntail;
        r = nr;
        h = nh;
        rb = nrb;
        k = nk;
        cnt = ncnt;
      }
    }
    // the CTA may not exit with copies in flight
    for (int i = issued > NS ? issued - NS : 0; i < issued; ++i)
      mbar_wait_bounded(&fullA[i % NS], (i / NS) & 1);
    for (int i = issued > NB ? issued - NB : 0; i < issued; ++i)
      mbar_wait_bounded(&fullB[i % NB], (i / NB) & 1);
  } else if (warp == kMmaWMma) {
    // ------------------------------------------------------------------ head MMA warp
    // The warp runs converged; one elected lane issues each tensor-core instruction. Per unit:
    // G (into the D2 columns of the unit's accumulator stage), then D1.
    int sver = -1;
    bool ok = true;
    for (int i = 0; i < n_my && ok; ++i) {
      const int s = i % NS, n = i / NS, sb = i % NB, ac = i % NA;
      ok = __all_sync(kFull, mbar_wait_bounded(&fullA[s], n & 1) &&
                                 mbar_wait_bounded(&fullB[sb], (i / NB) & 1));
      fence_proxy_async_smem();                    // cp.async data -> tensor-core reads
      const MmaInfo* inf = info(sb);
      const int U = min(inf->U, UC);
      const int lastu = inf->last;
      if (inf->first) ++sver;
      if (i >= NA) ok = ok && __all_sync(kFull, mbar_wait_bounded(&acc_empty[ac], ((i - NA) / NA) & 1));
      tc_fence_after();
      const uint32_t d1 = tmem + uint32_t(ac) * 128u, d2 = d1 + 64u;
      const uint32_t st = smem_u32(stage(s));
      if (ok) {
        // G[x][u] = x . k_u (M = 64 rows x of the q | k tile, N = 48 records), into the
        // columns that D2 overwrites once the coefficient warps have read G
        const uint32_t id0 = idesc_bf16_f32(64, UC);
        if (U > 0) {
#pragma unroll 1
          for (int kstep = 0; kstep < DK / 16; ++kstep) {
            const uint32_t ks = uint32_t(kstep >> 2), kk = uint32_t(kstep & 3);
            const uint64_t ax = sw128_kmajor_desc(st + ks * 8192u + kk * 32u);
            const uint64_t bk = sw128_kmajor_desc(st + L.ka_off + ks * (UC * 128u) + kk * 32u);
            umma_bf16_w(d2, ax, bk, id0, kstep != 0 ? 1u : 0u);
          }
        }
        umma_commit_w(&g_ready[ac]);
      }
      ok = ok && __all_sync(kFull, mbar_wait_bounded(sready, sver & 1));
      tc_fence_after();
      if (ok) {
        const uint32_t sa = tmem + 128u * NA;
        const uint32_t id1 = idesc_bf16_f32(128, 2 * NP);
#pragma unroll 1
        for (int kstep = 0; kstep < DK / 16; ++kstep) {
          const uint32_t ks = uint32_t(kstep >> 2), kk = uint32_t(kstep & 3);
          const uint64_t bx = sw128_kmajor_desc(st + ks * 8192u + kk * 32u);
          umma_bf16_ts_w(d1, sa + kstep * 8, bx, id1, kstep != 0 ? 1u : 0u);
          umma_bf16_ts_w(d1, sa + DK / 2 + kstep * 8, bx, id1, 1u);
        }
        // S_ctx is read by D1 only: after the last unit of a (request, head) it may be replaced
        if (lastu) umma_commit_w(sfree);
        umma_commit_w(&emptyA[s]);
        umma_commit_w(&acc_full[ac]);
      }
      if (!ok && lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 21, t);
    }
    // tensor memory is released only once the last MMAs have completed
    if (ok && n_my > 0) mbar_wait_bounded(&acc_full[(n_my - 1) % NA], ((n_my - 1) / NA) & 1);
    __syncwarp();
  } else if (warp == kMmaWTail) {
    // ------------------------------------------------------------------ tail MMA warp
    // Per unit, once its Cf is written: D2 = W^T Cf over the G columns.
    bool ok = true;
    for (int i = 0; i < n_my && ok; ++i) {
      const int s = i % NS, ac = i % NA;
      ok = __all_sync(kFull, mbar_wait_bounded(coef_ready, i & 1));
      tc_fence_after();
      if (ok) {
        const int U = min(info(i % NB)->U, UC);
        const uint32_t d2 = tmem + uint32_t(ac) * 128u + 64u;
        const uint32_t st = smem_u32(stage(s));
        const uint32_t id2 = idesc_bf16_f32_amn(128, 2 * NP);
#pragma unroll 1
        for (int kq = 0; kq < (U + 15) / 16; ++kq) {
          // the two 64-row blocks of the A operand: 1024 bytes apart, or (d_v = 64) the same
          // block twice
          const uint64_t ah = sw128_mnmajor_desc(st + L.wh_off + kq * 4096, DVB == 64 ? 0 : 1024, 2048);
          const uint64_t al = sw128_mnmajor_desc(st + L.wl_off + kq * 4096, DVB == 64 ? 0 : 1024, 2048);
          const uint64_t bh = sw128_kmajor_desc(smem_u32(CH) + kq * 32);
          const uint64_t bl = sw128_kmajor_desc(smem_u32(CL) + kq * 32);
          umma_bf16_w(d2, ah, bh, id2, kq != 0 ? 1u : 0u);
          umma_bf16_w(d2, al, bh, id2, 1u);
          umma_bf16_w(d2, ah, bl, id2, 1u);
        }
        umma_commit_w(coef_free);
        umma_commit_w(&emptyA[s]);
        umma_commit_w(&acc_full[ac]);
      }
      if (!ok && lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 24, t);
    }
    if (ok && n_my > 0) mbar_wait_bounded(&acc_full[(n_my - 1) % NA], ((n_my - 1) / NA) & 1);
    __syncwarp();
  } else if (warp == kMmaWPrep) {
    // ------------------------------------------------------------------ prep warp
    // Per unit, from the staged data only (nothing here waits for a tensor-core result, so the
    // warp runs ahead): the decay table, the per-position scalars and the append of alpha_p.
    for (int i = 0; i < n_my; ++i) {
      const int sb = i % NB, db = i & 1;
      bool ok = mbar_wait_bounded(&fullB[sb], (i / NB) & 1);
      if (i >= 2) ok = ok && mbar_wait_bounded(&dec_free[db], ((i - 2) >> 1) & 1);      // DEC[db] free
      if (!__all_sync(kFull, ok)) {
        if (lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 23, t);
        break;
      }
      const MmaInfo* inf = info(sb);
      const int r = inf->r, h = inf->h, n_pos = min(inf->n_pos, NP);
      // SC[sb] is free: the producers reuse the v slot sb (and this unit's fullB[sb], waited
      // above, completes) only after the epilogue of unit i - NB, the last reader, is done
      MmaScal* sc = SC + sb * NP;
      float* DEC = DEC0 + db * (NP * UC);
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
        if (inf->rb == 0) a.A[wnew] = alpha;
      }
      sc[p].e = e;
      sc[p].alpha = alpha;
      sc[p].beta = beta;
      sc[p].io = (r * a.B + b) * a.H + h;
      sc[p].wnew = wnew;
      sc[p].valid = valid ? 1 : 0;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&dec_ready[db]);
        mbar_arrive(&scal_ready[sb]);
      }
    }
  } else if (warp < kMmaWEpi) {
    // ------------------------------------------------------------------ coefficient warps
    const int sp = warp & 3;
    int sver = -1;
    __nv_bfloat16* kout = static_cast<__nv_bfloat16*>(a.Kr);
    for (int i = 0; i < n_my; ++i) {
      const int s = i % NS, n = i / NS, sb = i % NB, ac = i % NA, db = i & 1;
      bool ok = mbar_wait_bounded(&fullA[s], n & 1) && mbar_wait_bounded(&fullB[sb], (i / NB) & 1);
      const MmaInfo* inf = info(sb);
      const int r = inf->r, h = inf->h, U = min(inf->U, UC);
      if (inf->first) {
        ++sver;
        if (sver >= 1) ok = ok && mbar_wait_bounded(sfree, (sver - 1) & 1);
        if (!__all_sync(kFull, ok)) {
          if (lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 22, t);
          break;
        }
        // S_ctx rows 32 sp .. 32 sp + 31 (hi, then lo) into tensor memory; one row per lane, two
        // bf16 per 32-bit column, lower k in the low half (memory order); eight 16-byte loads in
        // flight per thread (the rows were prefetched into L2 by the producers)
        tc_fence_after();
        const int row = 32 * sp + lane;
        // d_v = 64: lanes 64..127 hold S_ctx rows 0..63 again
        const size_t srow = (size_t(r) * a.H + h) * MP + size_t(inf->rb) * 128 + (row % DVB);
        const uint32_t ta = tmem + (uint32_t(32 * sp) << 16) + 128u * NA;
#pragma unroll 1
        for (int c8 = 0; c8 < DK / 32; ++c8) {          // DK / 64 batches per half
          const int half = c8 / (DK / 64), cb = c8 % (DK / 64);
          const uint4* src = reinterpret_cast<const uint4*>((half ? S_lo : S_hi) + srow * DK) + 8 * cb;
          const uint4 w0[4] = {__ldg(src), __ldg(src + 1), __ldg(src + 2), __ldg(src + 3)};
          const uint4 w1[4] = {__ldg(src + 4), __ldg(src + 5), __ldg(src + 6), __ldg(src + 7)};
          tmem_st16(ta + half * (DK / 2) + (2 * cb) * 16, w0);
          tmem_st16(ta + half * (DK / 2) + (2 * cb + 1) * 16, w1);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sready);
      }
      // c0_p = k_p . q_p for the epilogue (fp32 sums of the staged bf16 rows): thread
      // (p, quarter) of the 128 coefficient threads takes a quarter of the row, then the four
      // partial sums are added across lanes; SC[sb] is free since fullB[sb] of this unit
      // completed (the prep warp's comment says why).
      {
        const int tc = 32 * sp + lane, p = tc >> 2, qd = tc & 3;
        const unsigned char* xs = stage(s);
        float c0 = 0.f;
#pragma unroll
        for (int j = 0; j < CR / 4; ++j) {
          const int c = qd * (CR / 4) + j, ks = c >> 3, cc = c & 7;
          const uint4 qv = *reinterpret_cast<const uint4*>(xs + ks * 8192 + p * 128 + ((cc ^ (p & 7)) << 4));
          const uint4 kv = *reinterpret_cast<const uint4*>(xs + ks * 8192 + (NP + p) * 128 +
                                                           ((cc ^ ((NP + p) & 7)) << 4));
          const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w}, kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const float2 qf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qw[e2]));
            const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kw[e2]));
            c0 = fmaf(qf.x, kf.x, c0);
            c0 = fmaf(qf.y, kf.y, c0);
          }
        }
        c0 += __shfl_xor_sync(kFull, c0, 1);
        c0 += __shfl_xor_sync(kFull, c0, 2);
        if (qd == 0) SC[sb * NP + p].c0 = c0;
        // append k_p (row block 0 only): the 128 threads copy the staged k rows (16-byte
        // chunks) into the records
        const int n_pos = inf->rb == 0 ? min(inf->n_pos, NP) : 0;
#pragma unroll
        for (int j = 0; j < CR / 4; ++j) {
          const int idx = tc * (CR / 4) + j, pk = idx / CR, c = idx % CR, nn = NP + pk;
          if (pk < n_pos) {
            const uint4 v = *reinterpret_cast<const uint4*>(xs + (c >> 3) * 8192 + nn * 128 +
                                                            (((c & 7) ^ (nn & 7)) << 4));
            const int wr = rec_row_hm(a, t - 1, r, h, inf->beam[pk]);
            *reinterpret_cast<uint4*>(kout + size_t(wr) * DK + c * 8) = v;
          }
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&scal_ready[sb]);
          mbar_arrive(&emptyA[s]);                   // done with the operand stage
        }
      }
      // the decay table (always waited, so these warps never run two units ahead of the prep
      // warp), G, and the previous unit's MMAs (waited at every unit so that the wait never
      // falls two phases behind the barrier)
      ok = ok && mbar_wait_bounded(&dec_ready[db], (i >> 1) & 1);
      ok = ok && mbar_wait_bounded(&g_ready[ac], (i / NA) & 1);
      if (i >= 1) ok = ok && mbar_wait_bounded(coef_free, (i - 1) & 1);
      if (!__all_sync(kFull, ok)) {
        if (lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 25, t);
        break;
      }
      tc_fence_after();
      if (U > 0) {
        // Cf = DEC * G, written as bf16 hi + lo, 16 records at a time. Lanes 0-15 hold rows
        // n = 16 sp + lane of G (the M = 64 layout puts rows 16 sp .. 16 sp + 15 in lanes 0-15 of
        // subpartition sp); lanes 16-31 take over records 8-15 of the same rows, so that every
        // lane converts and stores one 8-record chunk.
        const uint32_t tg = tmem + (uint32_t(32 * sp) << 16) + uint32_t(ac) * 128u + 64u;
        const int nrow = 16 * sp + (lane & 15), p = nrow & 31, q2 = lane >> 4;
        const float* dr = DEC0 + db * (NP * UC) + p * UC;
#pragma unroll 1
        for (int h16 = 0; h16 < UC / 16; ++h16) {
          if (16 * h16 >= U) break;                   // warp-uniform
          float gr[16];
          tmem_ld16(tg + 16u * h16, gr);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float lv = __shfl_up_sync(kFull, gr[8 + e], 16);
            if (lane >= 16) gr[e] = lv;
          }
          const int q = 2 * h16 + q2;
          const float4 d0 = *reinterpret_cast<const float4*>(dr + 8 * q);
          const float4 d1 = *reinterpret_cast<const float4*>(dr + 8 * q + 4);
          const float v[8] = {gr[0] * d0.x, gr[1] * d0.y, gr[2] * d0.z, gr[3] * d0.w,
                              gr[4] * d1.x, gr[5] * d1.y, gr[6] * d1.z, gr[7] * d1.w};
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 hi2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
            const float2 hf2 = __bfloat1622float2(hi2);
            const __nv_bfloat162 lo2 = __floats2bfloat162_rn(v[2 * e] - hf2.x, v[2 * e + 1] - hf2.y);
            hw[e] = *reinterpret_cast<const uint32_t*>(&hi2);
            lw[e] = *reinterpret_cast<const uint32_t*>(&lo2);
          }
          const uint32_t off = uint32_t(nrow) * 128u + uint32_t((q ^ (nrow & 7)) << 4);
          *reinterpret_cast<uint4*>(CH + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(CL + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&dec_free[db]);
        mbar_arrive(coef_ready);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    // thread = state row (tensor-memory lane); warp (sp, ph) = rows 32 sp.., positions 16 ph..
    const int ew = warp - kMmaWEpi, sp = warp & 3, ph = ew >> 2;
    const int row = 32 * sp + lane;
    // state row this lane finishes, and its positions: [16 ph, 16 ph + 16), or at d_v = 64
    // (lanes 64..127 repeat rows 0..63) [16 (sp / 2) + 8 ph, + 8)
    const int drow = row % DVB;
    const int pbase = DVB == 64 ? 16 * (sp >> 1) + 8 * ph : 16 * ph;
    constexpr int NPB = DVB == 64 ? 1 : 2;          // batches of 8 positions per warp
    const uint32_t tl = tmem + (uint32_t(32 * sp) << 16);
    __nv_bfloat16* Wb = reinterpret_cast<__nv_bfloat16*>(a.W);
    for (int i = 0; i < n_my; ++i) {
      const int sb = i % NB, ac = i % NA;
      bool ok = mbar_wait_bounded(&acc_full[ac], (i / NA) & 1);
      ok = ok && mbar_wait_bounded(&scal_ready[sb], (i / NB) & 1);
      if (!__all_sync(kFull, ok)) {
        if (lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 26, t);
        break;
      }
      tc_fence_after();
      const MmaScal* sc = SC + sb * NP;
      const unsigned char* Vb = vslot(sb);          // [2][32][128 B] sw128
      const MmaInfo* inf = info(sb);
      const int n_pos = min(inf->n_pos, NP), U = inf->U;
      const int orow = inf->rb * 128 + drow;          // row of o and of the w record
      const uint32_t base = tl + uint32_t(ac) * 128u;
#pragma unroll 1
      for (int pb = 0; pb < NPB; ++pb) {
        const int p0 = pbase + 8 * pb;
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
                  Vb + (drow >> 6) * (NP * 128) + pp * 128 + ((((drow & 63) >> 3) ^ (pp & 7)) << 4) +
                  (drow & 7) * 2));
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const int j = j4 + jj;
              if (p0 + j < n_pos) {
                const float uu = fmaf(sa[jj].x, k1[j], k2[j]);
                const float qq = fmaf(sa[jj].x, q1[j], q2[j]);
                const float w = sa[jj].z * (vv[jj] - sa[jj].y * uu);
                const float o = fmaf(sa[jj].y, qq, sa[jj].w * w);
                a.o[size_t(io[jj]) * DV + orow] = o;
                const __nv_bfloat16 whi = __float2bfloat16_rn(w);
                const __nv_bfloat16 wlo = __float2bfloat16_rn(w - __bfloat162float(whi));
                Wb[size_t(wn[jj]) * (2 * DV) + orow] = whi;
                Wb[size_t(wn[jj]) * (2 * DV) + DV + orow] = wlo;
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&acc_empty[ac]);
        mbar_arrive(&emptyB[sb]);
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

static bool mma_width(int d) { return d == 64 || d == 128 || d == 256; }

bool replay_mma_supported(int d_k, int d_v, int B, int T_max) {
  return mma_width(d_k) && mma_width(d_v) && T_max <= kMmaMaxT && B <= kMmaMaxB;
}

int replay_mma_unit_records(int d_k, int d_v) {
  switch (d_k * 1000 + d_v) {
    case 64064: return MmaCfg<64, 64>::UC;
    case 64128: return MmaCfg<64, 128>::UC;
    case 64256: return MmaCfg<64, 256>::UC;
    case 128064: return MmaCfg<128, 64>::UC;
    case 128128: return MmaCfg<128, 128>::UC;
    case 128256: return MmaCfg<128, 256>::UC;
    case 256064: return MmaCfg<256, 64>::UC;
    case 256128: return MmaCfg<256, 128>::UC;
    case 256256: return MmaCfg<256, 256>::UC;
  }
  return kUnitAnc;
}

size_t replay_mma_smem(int d_k, int d_v) {
  switch (d_k * 1000 + d_v) {
    case 64064: return mma_layout_of<64, 64>().bytes;
    case 64128: return mma_layout_of<64, 128>().bytes;
    case 64256: return mma_layout_of<64, 256>().bytes;
    case 128064: return mma_layout_of<128, 64>().bytes;
    case 128128: return mma_layout_of<128, 128>().bytes;
    case 128256: return mma_layout_of<128, 256>().bytes;
    case 256064: return mma_layout_of<256, 64>().bytes;
    case 256128: return mma_layout_of<256, 128>().bytes;
    case 256256: return mma_layout_of<256, 256>().bytes;
  }
  return ~size_t(0);
}

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

template <int DK, int DV>
static cudaError_t launch_mma_t(const void* S_hi, const void* S_lo, const StepArgs& a,
                                const UnitPlan& up, const CUtensorMap& mq, const CUtensorMap& mk,
                                const CUtensorMap& mv, const CUtensorMap& mkr, const CUtensorMap& mw,
                                int n_sm,
                                cudaStream_t stream) {
  const MmaLayout L = mma_layout_of<DK, DV>();
  auto kern = replay_mma_kernel<DK, DV>;
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = once_per_device(configured, [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(L.bytes));
  });
  if (e != cudaSuccess) return e;
  kern<<<n_sm, kMmaWarps * 32, L.bytes, stream>>>(static_cast<const __nv_bfloat16*>(S_hi),
                                                  static_cast<const __nv_bfloat16*>(S_lo), a, up,
                                                  mq, mk, mv, mkr, mw);
  return cudaGetLastError();
}

// S_hi, S_lo: the shared state split into bf16 hi + lo, [R*H][M_pad][d_k] (M_pad = d_v rounded
// up to a multiple of 128, zero rows past d_v). W records are stored
// as [hi plane | lo plane] bf16 rows of 2 d_v elements. mkr, mw from make_record_maps; the
// q, k and v maps are made here for this step's inputs.
cudaError_t launch_replay_mma(const StepArgs& a, const UnitPlan& up, const void* S_hi,
                              const void* S_lo, const CUtensorMap& mkr, const CUtensorMap& mw,
                              cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  const uint64_t rows = uint64_t(a.R) * a.B * a.H;
  if (!make_rows_map(&mq, a.q, rows, a.d_k, uint64_t(a.d_k) * 2) ||
      !make_rows_map(&mk, a.k, rows, a.d_k, uint64_t(a.d_k) * 2) ||
      !make_rows_map(&mv, a.v, rows, a.d_v, uint64_t(a.d_v) * 2))
    return cudaErrorInvalidValue;
  cudaError_t e = launch_plan_units(a, up, stream);
  if (e != cudaSuccess) return e;
  int n_sm = 0;
  e = device_sm_count(&n_sm);
  if (e != cudaSuccess) return e;
#define OLA_MMA_CASE(DK_, DV_)                                                              \
  case DK_ * 1000 + DV_:                                                                    \
    return launch_mma_t<DK_, DV_>(S_hi, S_lo, a, up, mq, mk, mv, mkr, mw, n_sm, stream);
  switch (a.d_k * 1000 + a.d_v) {
    OLA_MMA_CASE(64, 64)
    OLA_MMA_CASE(64, 128)
    OLA_MMA_CASE(64, 256)
    OLA_MMA_CASE(128, 64)
    OLA_MMA_CASE(128, 128)
    OLA_MMA_CASE(128, 256)
    OLA_MMA_CASE(256, 64)
    OLA_MMA_CASE(256, 128)
    OLA_MMA_CASE(256, 256)
  }
#undef OLA_MMA_CASE
  return cudaErrorInvalidValue;
}

}  // namespace ola
