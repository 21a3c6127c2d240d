// Chunked prompt prefill on tensor cores: d_k = d_v = 128, bf16 prompt.
//
// "Scientific Impact Assessment: OneLA", §1 Core Contribution: all beams of a request start
// from one recurrent state derived from the shared prompt. Token by token (alpha = exp(g)):
//     w_p = beta_p (v_p - alpha_p S k_p),    S <- alpha_p S + w_p k_p^T.
// The pages give only this token recurrence; the chunked form below is derived from it. For a
// chunk of C tokens j = 1..C entered with state S0, let G_j = g_1 + ... + g_j (inclusive) and
// a_j = exp(G_j). Unrolling the recurrence inside the chunk gives, for every token j,
//     w_j + sum_{m<j} L_jm w_m = R_j := beta_j (v_j - a_j S0 k_j),
//     L_jm = beta_j e^{G_j - G_m} (k_j . k_m)                              (m < j),
//     S_C  = a_C S0 + sum_j e^{G_C - G_j} w_j k_j^T.
// With T = (I + L)^-1 (unit lower triangular, a function of the chunk's keys and gates only):
//     Z = S0 K^T,   R = beta (V - a Z),   W = R T^T,   S_C = a_C S0 + (W D) K,
// D = diag(e^{G_C - G_j}); rows of S are independent (row i only meets v[i]). Every exponent
// is a difference G_j - G_m <= 0 or G <= 0, so no factor exceeds 1.
//
// One CTA per (request, head), one per SM (tensor memory: 384 of 512 columns):
//   warps 0-3, 10-13  two precompute groups taking alternate chunks, ahead of the state
//              chain: gates (prefix sums, a, D), K K^T on warp-level MMA from the key tile
//              (exact bf16 products), L, T in fp32 by 16 x 16 blocks (diagonal blocks by
//              forward substitution, then T_ba = -T_bb sum_{a <= c < b} L_bc T_ca by block
//              distance), T as bf16 hi + lo tiles
//   warps 4-7  state rows (thread = row = tensor-memory lane): R, W D, and the state entering
//              the next chunk (its bf16 hi + lo for Z, and a_C S for the accumulation)
//   warp 8     TMA: key and value tiles of each chunk, three stages
//   warp 9     tcgen05.mma: Z = S K^T (S hi + lo in tensor memory),
//              W = R T^T (three products of hi/lo parts), S += (W D) K (keys as MN-major B)
// fp32 values enter the tensor cores as hi = bf16(x) plus lo = bf16(x - hi) (about 16
// significant bits); the lo x lo product is dropped; keys are bf16 already and exact.
#include "ola_device.cuh"

namespace ola {

namespace {

constexpr int kC = 64;             // tokens per chunk
constexpr int kD = 128;            // d_k = d_v
constexpr int kStages = 3;
constexpr int kThreads = 448;
constexpr int kWRow = 4;           // first state-row warp
constexpr int kWTma = 8;
constexpr int kWMma = 9;
constexpr int kWPre1 = 10;         // first warp of the second precompute group
constexpr int kBarPre = 1;         // named barriers 1 and 2: the two precompute groups

// tensor memory columns (lane = state row)
constexpr uint32_t kTS = 0;        // S fp32, 128 columns
constexpr uint32_t kTSH = 128;     // S as bf16 hi, two per column (64 columns)
constexpr uint32_t kTSL = 192;     // S as bf16 lo
constexpr uint32_t kTZ = 256;      // Z, then W: fp32, one column per token (64)
constexpr uint32_t kTRH = 320;     // R, then W D: bf16 hi (32 columns)
constexpr uint32_t kTRL = 352;     // ... bf16 lo

// shared memory, offsets from a 1024-byte aligned base
constexpr uint32_t kTile = kC * kD * 2;                        // 16 KB: [2 col blocks][64][128 B]
constexpr uint32_t kTTile = kC * kC * 2;                       // 8 KB: [64][64] bf16, sw128
constexpr int kScFloats = 3 * kC + 4;                          // a, beta, D, a_C (+ pad)
constexpr int kLd = kC + 1;                                    // padded fp32 row of L
constexpr int kLdT = kC + 4;                                   // fp32 row of T (16-byte rows)
constexpr uint32_t kOffK = 0;                                  // keys, 128-byte swizzle
constexpr uint32_t kOffV = kOffK + kStages * kTile;            // values, no swizzle
constexpr uint32_t kOffT = kOffV + kStages * kTile;            // T hi, T lo per stage
constexpr uint32_t kOffSc = kOffT + kStages * 2 * kTTile;      // gate scalars per stage
constexpr uint32_t kOffGrp = kOffSc + kStages * kScFloats * 4; // per precompute group:
constexpr uint32_t kGL = 0;                                    //   L fp32 [64][65]
constexpr uint32_t kGTf = kGL + kC * kLd * 4;                  //   T fp32 [64][68]
constexpr uint32_t kGQ = kGTf + kC * kLdT * 4;                 //   block products [3][16][16]
constexpr uint32_t kGG = kGQ + 3 * 256 * 4;                    //   G_j [64] + a warp total
constexpr uint32_t kGrpBytes = kGG + (kC + 4) * 4;
constexpr uint32_t kOffBar = kOffGrp + 2 * kGrpBytes;
constexpr int kNumBars = 16;
constexpr uint32_t kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;   // + holder, alignment
static_assert(kOffBar % 8 == 0, "mbarriers need 8-byte alignment");
static_assert((kOffGrp + kGTf) % 16 == 0 && (kOffGrp + kGQ) % 16 == 0 && kGrpBytes % 16 == 0,
              "float4 rows of T and of the block products");
static_assert(kOffT % 1024 == 0 && kOffV % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

struct ChunkArgs {
  CUtensorMap mk;     // k [R][P][H][128] bf16: box 64 x 1 x 64 x 1, 128-byte swizzle
  CUtensorMap mv;     // v [R][P][H][128] bf16: same box, no swizzle
  const float* g;     // [R][P][H]
  const float* beta;  // [R][P][H]
  float* S;           // [R][H][128][128]
  int* err;           // 4 int32: code, detail, chunk
  int R, H, P, nch;
};

// Named barrier over `count` threads that also returns the AND of `v` over them.
__device__ __forceinline__ bool bar_and(int id, int count, bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(uint32_t(v)), "r"(id), "r"(count)
      : "memory");
  return out != 0;
}

// x (32 fp32, token order) as bf16 hi and lo words, two per word, the lower token in the low half.
__device__ __forceinline__ void split32(const float (&x)[32], uint4 (&hi)[4], uint4 (&lo)[4]) {
  uint32_t* hw = reinterpret_cast<uint32_t*>(hi);
  uint32_t* lw = reinterpret_cast<uint32_t*>(lo);
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
    const float2 hf = __bfloat1622float2(h2);
    const __nv_bfloat162 l2 = __floats2bfloat162_rn(x[2 * e] - hf.x, x[2 * e + 1] - hf.y);
    hw[e] = *reinterpret_cast<const uint32_t*>(&h2);
    lw[e] = *reinterpret_cast<const uint32_t*>(&l2);
  }
}

__device__ __forceinline__ void tmem_ld32(uint32_t t, float (&x)[32]) {
  float a[16], b[16];
  tmem_ld16(t, a);
  tmem_ld16(t + 16, b);
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    x[e] = a[e];
    x[16 + e] = b[e];
  }
}

__device__ __forceinline__ void tmem_st32(uint32_t t, const float (&x)[32]) {
  uint4 a[4], b[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    a[e] = make_uint4(__float_as_uint(x[4 * e]), __float_as_uint(x[4 * e + 1]),
                      __float_as_uint(x[4 * e + 2]), __float_as_uint(x[4 * e + 3]));
    b[e] = make_uint4(__float_as_uint(x[16 + 4 * e]), __float_as_uint(x[16 + 4 * e + 1]),
                      __float_as_uint(x[16 + 4 * e + 2]), __float_as_uint(x[16 + 4 * e + 3]));
  }
  tmem_st16(t, a);
  tmem_st16(t + 16, b);
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    prefill_chunk_kernel(const __grid_constant__ ChunkArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = align_smem_1024(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kOffBar);
  uint64_t* full = bar;              // [3] key and value tiles landed (TMA bytes)
  uint64_t* empty = bar + 3;         // [3] stage reusable: MMA commit + 4 state-row warps
  uint64_t* pre = bar + 6;           // [3] T tiles and gate scalars written: 4 precompute warps
  uint64_t* z_full = bar + 9;        // Z in tensor memory
  uint64_t* r_full = bar + 10;       // R hi/lo written (4 state-row warps)
  uint64_t* w_full = bar + 11;       // W in tensor memory
  uint64_t* y_full = bar + 12;       // W D hi/lo written (4 state-row warps)
  uint64_t* s_full = bar + 13;       // S updated
  uint64_t* shl_full = bar + 14;     // S hi/lo and a_C S written (4 state-row warps)
  uint64_t* mma_done = bar + 15;     // every MMA of the CTA completed
  uint32_t* holder = reinterpret_cast<uint32_t*>(bar + kNumBars);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = blockIdx.x / a.H, h = blockIdx.x % a.H;
  const int nch = a.nch;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 5);
      mbar_init(&pre[s], 4);
    }
    mbar_init(z_full, 1);
    mbar_init(r_full, 4);
    mbar_init(w_full, 1);
    mbar_init(y_full, 4);
    mbar_init(s_full, 1);
    mbar_init(shl_full, 4);
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == kWMma) tmem_alloc(holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  const uint32_t kbase = smem_u32(sm + kOffK);

  if (warp == kWTma) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&a.mk);
      prefetch_tmap(&a.mv);
      int issued = 0;
      for (int c = 0; c < nch; ++c) {
        const int s = c % kStages, n = c / kStages;
        if (n > 0 && !mbar_wait_bounded(&empty[s], (n - 1) & 1)) {
          report_error(a.err, OLA_ERR_TIMEOUT, 40, c);
          break;
        }
        mbar_arrive_expect_tx(&full[s], 2 * kTile);
        unsigned char* kt = sm + kOffK + s * kTile;
        unsigned char* vt = sm + kOffV + s * kTile;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          tma_load_4d(kt + x * 8192, &a.mk, &full[s], 64 * x, h, kC * c, r);
          tma_load_4d(vt + x * 8192, &a.mv, &full[s], 64 * x, h, kC * c, r);
        }
        issued = c + 1;
      }
      // the copies still in flight land before the CTA exits
      for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c)
        mbar_wait_bounded(&full[c % kStages], (c / kStages) & 1);
    }
  } else if (warp == kWMma) {
    // ---------------------------------------------------------------- MMA issue
    const uint32_t id_z = idesc_bf16_f32(128, kC);
    const uint32_t id_s = idesc_bf16_f32(128, kD) | (1u << 16);     // B (the keys) MN-major
    bool ok = true;
    for (int c = 0; c < nch && ok; ++c) {
      const int s = c % kStages, n = c / kStages;
      const uint32_t kb = kbase + s * kTile;
      // Z = S K^T: M = 128 state rows, N = 64 tokens, K = d_k; S as hi + lo from tensor memory
      ok = __all_sync(kFull, mbar_wait_bounded(&full[s], n & 1) &&
                                 mbar_wait_bounded(shl_full, c & 1));
      tc_fence_after();
      if (!ok) break;
#pragma unroll 1
      for (int ks = 0; ks < kD / 16; ++ks) {
        const uint64_t b = sw128_kmajor_desc(kb + (ks >> 2) * 8192 + (ks & 3) * 32);
        umma_bf16_ts_w(tmem + kTZ, tmem + kTSH + ks * 8, b, id_z, ks != 0);
        umma_bf16_ts_w(tmem + kTZ, tmem + kTSL + ks * 8, b, id_z, 1u);
      }
      umma_commit_w(z_full);
      // W = R T^T: M = 128, N = 64 tokens, K = 64 tokens; R_hi T_hi + R_hi T_lo + R_lo T_hi
      ok = __all_sync(kFull, mbar_wait_bounded(&pre[s], n & 1) && mbar_wait_bounded(r_full, c & 1));
      tc_fence_after();
      if (!ok) break;
      const uint32_t th = smem_u32(sm + kOffT + s * 2 * kTTile), tl = th + kTTile;
#pragma unroll 1
      for (int ks = 0; ks < kC / 16; ++ks) {
        const uint64_t bh = sw128_kmajor_desc(th + ks * 32), bl = sw128_kmajor_desc(tl + ks * 32);
        umma_bf16_ts_w(tmem + kTZ, tmem + kTRH + ks * 8, bh, id_z, ks != 0);
        umma_bf16_ts_w(tmem + kTZ, tmem + kTRH + ks * 8, bl, id_z, 1u);
        umma_bf16_ts_w(tmem + kTZ, tmem + kTRL + ks * 8, bh, id_z, 1u);
      }
      umma_commit_w(w_full);
      // S += (W D) K: M = 128, N = d_k, K = 64 tokens; the key tile read as an MN-major B
      // (128-byte rows of 64 key columns per token, column blocks 8 KB apart, 8 tokens per 1 KB)
      ok = __all_sync(kFull, mbar_wait_bounded(y_full, c & 1));
      tc_fence_after();
      if (!ok) break;
#pragma unroll 1
      for (int ks = 0; ks < kC / 16; ++ks) {
        const uint64_t b = sw128_mnmajor_desc(kb + ks * 2048, 8192, 1024);
        umma_bf16_ts_w(tmem + kTS, tmem + kTRH + ks * 8, b, id_s, 1u);
        umma_bf16_ts_w(tmem + kTS, tmem + kTRL + ks * 8, b, id_s, 1u);
      }
      umma_commit_w(s_full);
      umma_commit_w(&empty[s]);
    }
    if (!ok && lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 41, 0);
    // every MMA issued has completed before tensor memory is released
    umma_commit_w(mma_done);
    mbar_wait_bounded(mma_done, 0);
    __syncwarp();
  } else if (warp >= kWRow && warp < kWRow + 4) {
    // ---------------------------------------------------------------- state rows
    const int sp = warp & 3, i = 32 * sp + lane;
    const uint32_t tl = tmem + (uint32_t(32 * sp) << 16);
    {
      float z[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) z[e] = 0.f;
#pragma unroll 1
      for (int q = 0; q < 8; ++q) tmem_st32(tl + kTS + 32 * q, z);     // S, S hi, S lo = 0
      tmem_st_wait();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(shl_full);
    bool ok = true;
    for (int c = 0; c < nch; ++c) {
      const int s = c % kStages, n = c / kStages;
      const float* sc = reinterpret_cast<const float*>(sm + kOffSc + s * kScFloats * 4);
      ok = mbar_wait_bounded(&full[s], n & 1) && mbar_wait_bounded(&pre[s], n & 1) &&
           mbar_wait_bounded(z_full, c & 1);
      if (!__all_sync(kFull, ok)) break;
      tc_fence_after();
      // R_j = beta_j (v_j[i] - a_j Z_j)
      const __nv_bfloat16* vt =
          reinterpret_cast<const __nv_bfloat16*>(sm + kOffV + s * kTile + (i >> 6) * 8192) +
          (i & 63);
#pragma unroll 1
      for (int q = 0; q < 2; ++q) {
        float x[32];
        tmem_ld32(tl + kTZ + 32 * q, x);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const int j = 32 * q + 4 * e4;
          const float4 av = *reinterpret_cast<const float4*>(sc + j);
          const float4 bv = *reinterpret_cast<const float4*>(sc + kC + j);
          x[4 * e4] = bv.x * (__bfloat162float(vt[j * 64]) - av.x * x[4 * e4]);
          x[4 * e4 + 1] = bv.y * (__bfloat162float(vt[(j + 1) * 64]) - av.y * x[4 * e4 + 1]);
          x[4 * e4 + 2] = bv.z * (__bfloat162float(vt[(j + 2) * 64]) - av.z * x[4 * e4 + 2]);
          x[4 * e4 + 3] = bv.w * (__bfloat162float(vt[(j + 3) * 64]) - av.w * x[4 * e4 + 3]);
        }
        uint4 hi[4], lo[4];
        split32(x, hi, lo);
        tmem_st16(tl + kTRH + 16 * q, hi);
        tmem_st16(tl + kTRL + 16 * q, lo);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(r_full);
      // W D
      ok = mbar_wait_bounded(w_full, c & 1);
      if (!__all_sync(kFull, ok)) break;
      tc_fence_after();
#pragma unroll 1
      for (int q = 0; q < 2; ++q) {
        float x[32];
        tmem_ld32(tl + kTZ + 32 * q, x);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 dv = *reinterpret_cast<const float4*>(sc + 2 * kC + 32 * q + 4 * e4);
          x[4 * e4] *= dv.x;
          x[4 * e4 + 1] *= dv.y;
          x[4 * e4 + 2] *= dv.z;
          x[4 * e4 + 3] *= dv.w;
        }
        uint4 hi[4], lo[4];
        split32(x, hi, lo);
        tmem_st16(tl + kTRH + 16 * q, hi);
        tmem_st16(tl + kTRL + 16 * q, lo);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(y_full);
        mbar_arrive(&empty[s]);                      // done with this stage's values and scalars
      }
      // the state leaving the chunk: bf16 hi + lo for the next Z, a_C S for the next update
      const bool last = c + 1 == nch;
      const int s1 = (c + 1) % kStages;
      ok = mbar_wait_bounded(s_full, c & 1);
      if (!last) ok = ok && mbar_wait_bounded(&pre[s1], ((c + 1) / kStages) & 1);
      if (!__all_sync(kFull, ok)) break;
      tc_fence_after();
      if (!last) {
        // hi + lo for the next Z first (the chain waits on them), then a_C S for the next
        // accumulation, which overlaps the next Z
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          float x[32];
          tmem_ld32(tl + kTS + 32 * q, x);
          uint4 hi[4], lo[4];
          split32(x, hi, lo);
          tmem_st16(tl + kTSH + 16 * q, hi);
          tmem_st16(tl + kTSL + 16 * q, lo);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(shl_full);
        const float aC =
            reinterpret_cast<const float*>(sm + kOffSc + s1 * kScFloats * 4)[3 * kC];
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          float x[32];
          tmem_ld32(tl + kTS + 32 * q, x);
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] *= aC;
          tmem_st32(tl + kTS + 32 * q, x);
        }
        tmem_st_wait();
      } else {
        float* dst = a.S + ((size_t(r) * a.H + h) * kD + i) * size_t(kD);
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          float x[32];
          tmem_ld32(tl + kTS + 32 * q, x);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            reinterpret_cast<float4*>(dst + 32 * q)[e] =
                make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
        }
      }
    }
    if (!ok && lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 42, 0);
  } else {
    // ---------------------------------------------------------------- per-chunk precompute
    // group grp takes chunks grp, grp + 2, ...; ptid = thread, pw = warp within the group
    const int grp = warp >= kWPre1 ? 1 : 0;
    const int ptid = tid - 32 * (grp ? kWPre1 : 0), pw = ptid >> 5, pbar = kBarPre + grp;
    unsigned char* gb = sm + kOffGrp + grp * kGrpBytes;
    float* Lm = reinterpret_cast<float*>(gb + kGL);
    float* Tf = reinterpret_cast<float*>(gb + kGTf);
    float* Qb = reinterpret_cast<float*>(gb + kGQ);
    float* Gs = reinterpret_cast<float*>(gb + kGG);
    // gates of chunk c (tokens past P: g = 0, beta = 0, an identity step), loaded a chunk ahead
    auto load_gates = [&](int c, float& gv, float& bv) {
      gv = 0.f;
      bv = 0.f;
      const int p = kC * c + ptid;
      if (ptid < kC && c < nch && p < a.P) {
        const size_t ix = (size_t(r) * a.P + p) * a.H + h;
        gv = __ldg(a.g + ix);
        bv = __ldg(a.beta + ix);
      }
    };
    float gj, bj;
    load_gates(grp, gj, bj);
    for (int c = grp; c < nch; c += 2) {
      const int s = c % kStages, n = c / kStages;
      float* sc = reinterpret_cast<float*>(sm + kOffSc + s * kScFloats * 4);
      bool ok = n == 0 || mbar_wait_bounded(&empty[s], (n - 1) & 1);
      if (!bar_and(pbar, 128, ok)) {
        if (ptid == 0) report_error(a.err, OLA_ERR_TIMEOUT, 43, c);
        break;
      }
      // gates: G_j by an inclusive scan (tokens 0-31 in the group's warp 0, 32-63 in its warp 1)
      float G = gj;
      const float bcur = bj;
      load_gates(c + 2, gj, bj);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(kFull, G, o);
        if (lane >= o) G += y;
      }
      if (ptid == 31) Gs[kC] = G;
      named_bar_sync(pbar, 128);
      if (ptid >= 32 && ptid < kC) G += Gs[kC];
      if (ptid < kC) Gs[ptid] = G;
      named_bar_sync(pbar, 128);
      const float GC = Gs[kC - 1];
      if (ptid < kC) {
        sc[ptid] = expf(G);
        sc[kC + ptid] = bcur;
        sc[2 * kC + ptid] = expf(GC - G);
      }
      if (ptid == 0) sc[3 * kC] = expf(GC);
      // K K^T rows 16 w .. 16 w + 15 (group warp w) on warp-level MMA from the swizzled key
      // tile, the 16-column tiles up to the diagonal only, and L from it (entries on or above
      // the diagonal are never read)
      ok = mbar_wait_bounded(&full[s], n & 1);
      if (!bar_and(pbar, 128, ok)) {
        if (ptid == 0) report_error(a.err, OLA_ERR_TIMEOUT, 44, c);
        break;
      }
      {
        const uint32_t kt = smem_u32(sm + kOffK + s * kTile);
        // byte of the 8 keys columns x .. x + 7 of token t in the tile
        auto kaddr = [&](int t, int x) {
          return kt + uint32_t(x >> 6) * 8192u + uint32_t(t) * 128u +
                 uint32_t((((x & 63) >> 3) ^ (t & 7)) << 4);
        };
        const int jb = pw;
        uint32_t af[8][4];
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          ldsm_x4(kaddr(16 * jb + (lane & 15), 16 * ks + (lane >> 4) * 8), af[ks][0], af[ks][1],
                  af[ks][2], af[ks][3]);
        const int j0 = 16 * jb + (lane >> 2), j1 = j0 + 8, cq = 2 * (lane & 3);
        const float G0 = Gs[j0], G1 = Gs[j1], b0 = sc[kC + j0], b1 = sc[kC + j1];
        const int bt = ((lane >> 3) >> 1) * 8 + (lane & 7), bx = ((lane >> 3) & 1) * 8;
        // the column tiles of the row block accumulate side by side: 2 (jb + 1) independent
        // MMA chains of 8 steps instead of one long chain
        float d[4][2][4];
#pragma unroll
        for (int mp = 0; mp < 4; ++mp)
#pragma unroll
          for (int e = 0; e < 4; ++e) d[mp][0][e] = d[mp][1][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
          for (int mp = 0; mp < 4; ++mp) {
            if (mp <= jb) {                              // warp-uniform
              uint32_t b00, b01, b10, b11;
              ldsm_x4(kaddr(16 * mp + bt, 16 * ks + bx), b00, b01, b10, b11);
              mma_16816_bf16(d[mp][0], af[ks][0], af[ks][1], af[ks][2], af[ks][3], b00, b01);
              mma_16816_bf16(d[mp][1], af[ks][0], af[ks][1], af[ks][2], af[ks][3], b10, b11);
            }
          }
        }
#pragma unroll
        for (int mp = 0; mp < 4; ++mp) {
          if (mp > jb) break;
          const float* d0 = d[mp][0];
          const float* d1 = d[mp][1];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int m = 16 * mp + cq + e, m8 = m + 8;
            const float Gm = Gs[m], Gm8 = Gs[m8];
            Lm[j0 * kLd + m] = m < j0 ? b0 * __expf(G0 - Gm) * d0[e] : 0.f;
            Lm[j1 * kLd + m] = m < j1 ? b1 * __expf(G1 - Gm) * d0[2 + e] : 0.f;
            Lm[j0 * kLd + m8] = m8 < j0 ? b0 * __expf(G0 - Gm8) * d1[e] : 0.f;
            Lm[j1 * kLd + m8] = m8 < j1 ? b1 * __expf(G1 - Gm8) * d1[2 + e] : 0.f;
          }
        }
      }
      named_bar_sync(pbar, 128);
      // T = (I + L)^-1: the four 16 x 16 diagonal blocks by forward substitution (thread =
      // column), then T_ba = -T_bb sum_{a <= c < b} L_bc T_ca by block distance b - a
      if (ptid < kC) {
        const int o = 16 * (ptid >> 4), m = ptid & 15;
        // right-looking: once x[ii] is final it updates every later row (a chain of 15 steps)
        float x[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) x[jj] = jj == m ? 1.f : 0.f;
#pragma unroll
        for (int ii = 0; ii < 15; ++ii) {
#pragma unroll
          for (int jj = ii + 1; jj < 16; ++jj) x[jj] -= Lm[(o + jj) * kLd + o + ii] * x[ii];
        }
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) Tf[(o + jj) * kLdT + o + m] = x[jj];
      }
      named_bar_sync(pbar, 128);
      // task = (block pair, row y, 4 columns x0..x0+3)
#pragma unroll 1
      for (int dl = 1; dl < 4; ++dl) {
        const int ntask = (4 - dl) * 64;
        for (int o = ptid; o < ntask; o += 128) {
          const int ab = o >> 6, bb = ab + dl, y = (o >> 2) & 15, x0 = (o & 3) * 4;
          const float* lrow = Lm + (16 * bb + y) * kLd;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
          for (int cb = ab; cb < bb; ++cb) {
#pragma unroll
            for (int z = 0; z < 16; ++z) {
              const float l = lrow[16 * cb + z];
              const float4 t =
                  *reinterpret_cast<const float4*>(Tf + (16 * cb + z) * kLdT + 16 * ab + x0);
              acc.x += l * t.x;
              acc.y += l * t.y;
              acc.z += l * t.z;
              acc.w += l * t.w;
            }
          }
          *reinterpret_cast<float4*>(Qb + (ab * 16 + y) * 16 + x0) = acc;
        }
        named_bar_sync(pbar, 128);
        for (int o = ptid; o < ntask; o += 128) {
          const int ab = o >> 6, bb = ab + dl, y = (o >> 2) & 15, x0 = (o & 3) * 4;
          // T_bb row y (zeros past the diagonal)
          const float* trow = Tf + (16 * bb + y) * kLdT + 16 * bb;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int z = 0; z < 16; ++z) {
            const float tz = trow[z];
            const float4 q = *reinterpret_cast<const float4*>(Qb + (ab * 16 + z) * 16 + x0);
            acc.x -= tz * q.x;
            acc.y -= tz * q.y;
            acc.z -= tz * q.z;
            acc.w -= tz * q.w;
          }
          *reinterpret_cast<float4*>(Tf + (16 * bb + y) * kLdT + 16 * ab + x0) = acc;
        }
        named_bar_sync(pbar, 128);
      }
      // T as bf16 hi and lo, K-major tiles with the 128-byte swizzle: thread = half a row
      {
        const int jr = ptid >> 1, hf = ptid & 1;
        unsigned char* thi = sm + kOffT + s * 2 * kTTile;
        unsigned char* tlo = thi + kTTile;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int q = 4 * hf + qq;
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int m0 = 8 * q + 2 * e;
            const float t0 = m0 <= jr ? Tf[jr * kLdT + m0] : 0.f;
            const float t1 = m0 + 1 <= jr ? Tf[jr * kLdT + m0 + 1] : 0.f;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(t0, t1);
            const float2 hf2 = __bfloat1622float2(h2);
            const __nv_bfloat162 l2 = __floats2bfloat162_rn(t0 - hf2.x, t1 - hf2.y);
            hw[e] = *reinterpret_cast<const uint32_t*>(&h2);
            lw[e] = *reinterpret_cast<const uint32_t*>(&l2);
          }
          const uint32_t off = uint32_t(jr) * 128u + uint32_t((q ^ (jr & 7)) << 4);
          *reinterpret_cast<uint4*>(thi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(tlo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pre[s]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------- host side

namespace {

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                             const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                             const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                             CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn prompt_encoder() {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  }
  return fn;
}

// [R][P][H][128] bf16 as a 4-D map (column, head, token, request); a 64 x 1 x 64 x 1 box is
// one 64-column block of 64 consecutive tokens of one (request, head). Tokens past P read 0.
bool make_prompt_map(CUtensorMap* map, const void* base, int R, int P, int H, bool swizzle) {
  EncodeFn fn = prompt_encoder();
  if (!fn) return false;
  cuuint64_t dims[4] = {cuuint64_t(kD), cuuint64_t(H), cuuint64_t(P), cuuint64_t(R)};
  cuuint64_t strides[3] = {cuuint64_t(kD) * 2, cuuint64_t(H) * kD * 2,
                           cuuint64_t(P) * H * kD * 2};
  cuuint32_t box[4] = {64, 1, kC, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

bool prefill_chunk_supported(int d_k, int d_v, int in_dtype, const void* k, const void* v) {
  return d_k == kD && d_v == kD && in_dtype == OLA_BF16 &&
         (reinterpret_cast<uintptr_t>(k) & 15) == 0 && (reinterpret_cast<uintptr_t>(v) & 15) == 0;
}

// P >= 1. err: 4 device int32, zeroed by the caller.
cudaError_t launch_prefill_chunk(int R, int H, int P, const void* k, const void* v,
                                 const float* g, const float* beta, float* S_out, int* err,
                                 cudaStream_t stream) {
  ChunkArgs a;
  if (!make_prompt_map(&a.mk, k, R, P, H, true) || !make_prompt_map(&a.mv, v, R, P, H, false))
    return cudaErrorInvalidValue;
  a.g = g;
  a.beta = beta;
  a.S = S_out;
  a.err = err;
  a.R = R;
  a.H = H;
  a.P = P;
  a.nch = (P + kC - 1) / kC;
  cudaError_t e = cudaFuncSetAttribute(prefill_chunk_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  prefill_chunk_kernel<<<unsigned(R) * unsigned(H), kThreads, kSmemBytes, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace ola
