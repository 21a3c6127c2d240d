// Chunked prompt prefill on tensor cores: d_k = d_v = 128, bf16 prompt.
//
// "Scientific Impact Assessment: OneLA", §1 Core Contribution: all beams of a request start
// from one recurrent state derived from the shared prompt. Token by token (alpha = exp(g)):
//     w_p = beta_p (v_p - alpha_p S k_p),    S <- alpha_p S + w_p k_p^T.
// The pages give only this token recurrence; the chunked form below is derived from it. For a
// chunk of C tokens j = 1..C entered with state S0, let G_j = g_1 + ... + g_j (inclusive),
// a_j = exp(G_j) and D_j = exp(G_C - G_j). Unrolling the recurrence inside the chunk gives
//     w_j + sum_{m<j} beta_j e^{G_j - G_m} (k_j . k_m) w_m = beta_j (v_j - a_j S0 k_j),
//     S_C = a_C S0 + sum_j D_j w_j k_j^T.
// The decay factors of the triangular system are a diagonal similarity, E A E^-1 with
// E = diag(e^{G_j}) and A = I + diag(beta) K~ (K~ the strictly lower part of K K^T), so with
// T = A^-1 (unit lower triangular, no exponentials) w_m = sum_j e^{G_m - G_j} T_mj (...)_j.
// Collecting the chunk's decayed writes Y = [D_m w_m]_m (d_v x C), every exponential becomes a
// per-token scalar:
//     Y = U + S0 N,   U = V^T M1,   N = K^T M2,
//     M1_jm = beta_j D_j T_mj,   M2_jm = -a_C beta_j T_mj = -a_j M1_jm,
// so the state meets the chunk in one product, and S_C = a_C S0 + Y K. U and N depend only on
// the chunk's inputs and are formed off the state chain; no exponent is positive.
//
// One CTA per (request, head), one per SM (tensor memory: all 512 columns):
//   warp 14    tcgen05.mma: the Gram matrix K K^T of each chunk (exact bf16 products) once
//              its key tile has landed
//   warp 15    tcgen05.mma: N of each chunk once its M2 tiles are written
//   warps 0-3, 10-13  two precompute groups taking alternate chunks, ahead of the state chain:
//              gates (prefix sums, beta, beta D, -a), L = diag(beta) K~ from the Gram matrix,
//              T = (I + L)^-1 in fp32 by 16 x 16 blocks (diagonal blocks by forward
//              substitution, the others by block products over two halves of 32),
//              M1 and M2 as bf16 hi + lo tiles
//   warp 9     tcgen05.mma, the chain: P = U + S N (S hi + lo in tensor memory), S += Y K
//              (keys as MN-major B), then U of the next chunk into P's columns
//   warps 4-7  state rows (thread = row = tensor-memory lane): Y = P as bf16 hi + lo, the
//              state leaving the chunk (its bf16 hi + lo for P, and a_C S for the accumulation),
//              and, while S is updated, the next chunk's N as bf16 hi + lo tiles
//   warp 8     TMA: key and value tiles of each chunk, three stages
// Per chunk the chain is P, the Y split, S += Y K and the state's split. fp32 values enter the
// tensor cores as hi = bf16(x) plus lo = bf16(x - hi) (about 16 significant bits); the lo x lo
// product is dropped; keys and values are bf16 already and exact.
#include "ola_device.cuh"

namespace ola {

namespace {

constexpr int kC = 64;             // tokens per chunk
constexpr int kD = 128;            // d_k = d_v
constexpr int kStages = 3;
constexpr int kThreads = 512;
constexpr int kWRow = 4;           // first state-row warp
constexpr int kWTma = 8;
constexpr int kWMma = 9;
constexpr int kWPre1 = 10;         // first warp of the second precompute group
constexpr int kWGram = 14;
constexpr int kWN = 15;
constexpr int kBarPre = 1;         // named barriers 1 and 2: the two precompute groups

// tensor memory columns
constexpr uint32_t kTS = 0;        // S fp32, 128 columns (lane = state row)
constexpr uint32_t kTSH = 128;     // S as bf16 hi, two per column (64 columns)
constexpr uint32_t kTSL = 192;     // S as bf16 lo
constexpr uint32_t kTP = 256;      // P = U + S N = Y: fp32, one column per token (64)
constexpr uint32_t kTYH = 320;     // Y as bf16 hi (32 columns)
constexpr uint32_t kTYL = 352;     // ... bf16 lo
constexpr uint32_t kTN = 384;      // N fp32 (lane = key column, one column per token)
constexpr uint32_t kTG = 448;      // K K^T fp32 (lanes 0-63 = token)

// shared memory, offsets from a 1024-byte aligned base
constexpr uint32_t kTile = kC * kD * 2;                        // 16 KB: [2 col blocks][64][128 B]
constexpr uint32_t kMTile = kC * kC * 2;                       // 8 KB: [64][64] bf16, sw128
constexpr uint32_t kNTile = kD * kC * 2;                       // 16 KB: [128 key columns][64]
constexpr int kScFloats = 3 * kC + 4;                          // beta, beta D, -a, a_C
constexpr int kLd = kC + 4;                                    // fp32 row of L (16-byte rows)
constexpr int kLdT = kC + 4;                                   // fp32 row of T (16-byte rows)
constexpr uint32_t kOffK = 0;                                  // keys, 128-byte swizzle
constexpr uint32_t kOffV = kOffK + kStages * kTile;            // values, 128-byte swizzle
constexpr uint32_t kOffN = kOffV + kStages * kTile;            // N hi, N lo (one chunk)
constexpr uint32_t kOffSc = kOffN + 2 * kNTile;                // gate scalars per stage
constexpr uint32_t kOffGrp = kOffSc + 3072;                    // per precompute group:
constexpr uint32_t kGL = 0;                                    //   L fp32 [64][68], then M1 hi, lo
constexpr uint32_t kGTf = 17408;                               //   T fp32 [64][68], then M2 hi, lo
constexpr uint32_t kGQ = kGTf + kC * kLdT * 4;                 //   block products [4][16][16]
constexpr uint32_t kGG = kGQ + 4 * 256 * 4;                    //   G_j [64] + a warp total
constexpr uint32_t kGrpBytes = 39936;
constexpr uint32_t kOffBar = kOffGrp + 2 * kGrpBytes;
constexpr int kNumBars = 23;
constexpr uint32_t kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;   // + holder, alignment
static_assert(kStages * kScFloats * 4 <= 3072, "gate scalars");
static_assert(kC * kLd * 4 <= kGTf && 2 * kMTile <= kC * kLd * 4, "L region holds M1 hi + lo");
static_assert(2 * kMTile <= kC * kLdT * 4, "T region holds M2 hi + lo");
static_assert(kGG + (kC + 4) * 4 <= kGrpBytes && kGrpBytes % 1024 == 0, "group region");
static_assert(kOffGrp % 1024 == 0 && kGTf % 1024 == 0 && kOffN % 1024 == 0 &&
              kOffV % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert((kOffGrp + kGQ) % 16 == 0 && (kOffGrp + kGTf) % 16 == 0,
              "float4 rows of T and of the block products");
static_assert(kOffBar % 8 == 0, "mbarriers need 8-byte alignment");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

struct ChunkArgs {
  CUtensorMap mk;     // k [R][P][H][128] bf16: box 64 x 1 x 64 x 1, 128-byte swizzle
  CUtensorMap mv;     // v [R][P][H][128] bf16: same box and swizzle
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

// hi = bf16(x), lo = bf16(x - hi) for a pair, packed two per word (the first in the low half).
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h2 = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h2);
  const __nv_bfloat162 l2 = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h2);
  lo = *reinterpret_cast<const uint32_t*>(&l2);
}

// x (32 fp32, token order) as bf16 hi and lo words, two per word, the lower token in the low half.
__device__ __forceinline__ void split32(const float (&x)[32], uint4 (&hi)[4], uint4 (&lo)[4]) {
  uint32_t* hw = reinterpret_cast<uint32_t*>(hi);
  uint32_t* lw = reinterpret_cast<uint32_t*>(lo);
#pragma unroll
  for (int e = 0; e < 16; ++e) split2(x[2 * e], x[2 * e + 1], hw[e], lw[e]);
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

// N of chunk c (in tensor memory, lane = key column) to the MN-major hi/lo tiles of the chain's
// P product: row = key column i, 64 tokens in 128 bytes, 128-byte swizzle. Called by the
// state-row warps between their own steps (the previous P product has read the tiles); out of
// line, so that its three call sites share one copy of the code.
static __device__ __noinline__ bool convert_n(uint32_t tl, unsigned char* th, int i,
                                              uint64_t* n_full, uint64_t* n_ready, int c) {
  if (!__all_sync(kFull, mbar_wait_bounded(n_full, c & 1))) return false;
  tc_fence_after();
  unsigned char* tlo = th + kNTile;
#pragma unroll 1
  for (int hf = 0; hf < 2; ++hf) {                   // tokens 32 hf .. 32 hf + 31
    float x[32];
    tmem_ld32(tl + kTN + 32 * hf, x);
    uint4 hi[4], lo[4];
    split32(x, hi, lo);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t off = uint32_t(((4 * hf + q) ^ (i & 7)) << 4);
      *reinterpret_cast<uint4*>(th + off) = hi[q];
      *reinterpret_cast<uint4*>(tlo + off) = lo[q];
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(n_ready);
  return true;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    prefill_chunk_kernel(const __grid_constant__ ChunkArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = align_smem_1024(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kOffBar);
  uint64_t* full = bar;              // [3] key and value tiles landed (TMA bytes)
  uint64_t* empty = bar + 3;         // [3] stage reusable: chain MMA commit + 4 state-row warps
  uint64_t* pre = bar + 6;           // [3] M1, M2 tiles and gate scalars written (4 warps)
  uint64_t* kk_full = bar + 9;       // [2] Gram matrix of the group's chunk in tensor memory
  uint64_t* kk_free = bar + 11;      // Gram matrix read (2 warps)
  uint64_t* n_full = bar + 12;       // N of the next chunk in tensor memory
  uint64_t* m_free = bar + 13;       // [2] the group's M1, M2 tiles read (U and N commits)
  uint64_t* n_ready = bar + 15;      // N hi/lo tiles written (4 state-row warps)
  uint64_t* p_full = bar + 16;       // P in tensor memory
  uint64_t* y_full = bar + 17;       // Y hi/lo written (4 state-row warps)
  uint64_t* s_full = bar + 18;       // S updated
  uint64_t* shl_full = bar + 19;     // S hi/lo written (4 state-row warps)
  uint64_t* mma_done = bar + 20;     // every chain MMA completed
  uint64_t* gram_done = bar + 21;    // every Gram MMA completed
  uint64_t* n_done = bar + 22;       // every N MMA completed
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
    for (int g = 0; g < 2; ++g) {
      mbar_init(&kk_full[g], 1);
      mbar_init(&m_free[g], 2);
    }
    mbar_init(n_full, 1);
    mbar_init(n_ready, 4);
    mbar_init(kk_free, 2);
    mbar_init(p_full, 1);
    mbar_init(y_full, 4);
    mbar_init(s_full, 1);
    mbar_init(shl_full, 4);
    mbar_init(mma_done, 1);
    mbar_init(gram_done, 1);
    mbar_init(n_done, 1);
    fence_barrier_init();
  }
  if (warp == kWMma) tmem_alloc(holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  const uint32_t kbase = smem_u32(sm + kOffK);
  const uint32_t vbase = smem_u32(sm + kOffV);

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
  } else if (warp == kWGram) {
    // ---------------------------------------------------------------- Gram matrix
    // K K^T: M = 128 (rows 0-63 the chunk's tokens; rows 64-127 read whatever lies past the
    // tile in shared memory and are never used), N = 64 tokens, K = d_k
    const uint32_t id_g = idesc_bf16_f32(128, kC);
    bool ok = true;
    for (int c = 0; c < nch && ok; ++c) {
      const int s = c % kStages;
      ok = __all_sync(kFull, mbar_wait_bounded(&full[s], (c / kStages) & 1) &&
                                 (c == 0 || mbar_wait_bounded(kk_free, (c - 1) & 1)));
      tc_fence_after();
      if (!ok) break;
      const uint32_t kb = kbase + s * kTile;
#pragma unroll 1
      for (int ks = 0; ks < kD / 16; ++ks) {
        const uint64_t d = sw128_kmajor_desc(kb + (ks >> 2) * 8192 + (ks & 3) * 32);
        umma_bf16_w(tmem + kTG, d, d, id_g, ks != 0 ? 1u : 0u);
      }
      umma_commit_w(&kk_full[c & 1]);
    }
    if (!ok && lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 45, 0);
    umma_commit_w(gram_done);
    mbar_wait_bounded(gram_done, 0);
    __syncwarp();
  } else if (warp == kWN) {
    // ---------------------------------------------------------------- N = K^T M2
    // A the key tile read MN-major (d_k along M), B the chunk's M2 tiles; once they are written
    // and the previous N has left tensor memory
    const uint32_t id_n = idesc_bf16_f32_amn(128, kC);
    bool ok = true;
    for (int c = 0; c < nch && ok; ++c) {
      ok = __all_sync(kFull, mbar_wait_bounded(&pre[c % kStages], (c / kStages) & 1) &&
                                 (c == 0 || mbar_wait_bounded(n_ready, (c - 1) & 1)));
      tc_fence_after();
      if (!ok) break;
      const uint32_t kb = kbase + (c % kStages) * kTile;
      const uint32_t mh = smem_u32(sm + kOffGrp + (c & 1) * kGrpBytes + kGTf), ml = mh + kMTile;
#pragma unroll 1
      for (int ks = 0; ks < kC / 16; ++ks) {
        const uint64_t ak = sw128_mnmajor_desc(kb + ks * 2048, 8192, 1024);
        umma_bf16_w(tmem + kTN, ak, sw128_kmajor_desc(mh + ks * 32), id_n, ks != 0 ? 1u : 0u);
        umma_bf16_w(tmem + kTN, ak, sw128_kmajor_desc(ml + ks * 32), id_n, 1u);
      }
      umma_commit_w(n_full);
      umma_commit_w(&m_free[c & 1]);
    }
    if (!ok && lane == 0) report_error(a.err, OLA_ERR_TIMEOUT, 47, 0);
    umma_commit_w(n_done);
    mbar_wait_bounded(n_done, 0);
    __syncwarp();
  } else if (warp == kWMma) {
    // ---------------------------------------------------------------- chain MMA issue
    const uint32_t id_u = idesc_bf16_f32_amn(128, kC);              // U: A MN-major
    const uint32_t id_p = idesc_bf16_f32(128, kC) | (1u << 16);     // P: B (N tiles) MN-major
    const uint32_t id_s = idesc_bf16_f32(128, kD) | (1u << 16);     // S: B (the keys) MN-major
    const uint32_t nh = smem_u32(sm + kOffN), nl = nh + kNTile;
    // U = V^T M1 of chunk c1 into P's columns (A: the value tile read MN-major, d_v along M)
    auto issue_u = [&](int c1) -> bool {
      const int s1 = c1 % kStages;
      const uint32_t par = uint32_t(c1 / kStages) & 1u;
      const bool ok1 = __all_sync(kFull, mbar_wait_bounded(&pre[s1], par) &&
                                             mbar_wait_bounded(&full[s1], par));
      tc_fence_after();
      if (!ok1) return false;
      const uint32_t vb = vbase + s1 * kTile;
      const uint32_t mh = smem_u32(sm + kOffGrp + (c1 & 1) * kGrpBytes + kGL), ml = mh + kMTile;
#pragma unroll 1
      for (int ks = 0; ks < kC / 16; ++ks) {
        const uint64_t av = sw128_mnmajor_desc(vb + ks * 2048, 8192, 1024);
        umma_bf16_w(tmem + kTP, av, sw128_kmajor_desc(mh + ks * 32), id_u, ks != 0 ? 1u : 0u);
        umma_bf16_w(tmem + kTP, av, sw128_kmajor_desc(ml + ks * 32), id_u, 1u);
      }
      umma_commit_w(&m_free[c1 & 1]);
      return true;
    };
    // step c: the chain of chunk c (c >= 0), then U of chunk c + 1 (one call site for U)
    bool ok = true;
    for (int c = -1; c < nch && ok; ++c) {
      if (c >= 0) {
        const int s = c % kStages;
        const uint32_t kb = kbase + s * kTile;
        // P += S N: M = 128 state rows, N = 64 tokens, K = d_k; S_hi N_hi + S_hi N_lo + S_lo N_hi
        ok = __all_sync(kFull, mbar_wait_bounded(n_ready, c & 1) &&
                                   mbar_wait_bounded(shl_full, c & 1));
        tc_fence_after();
        if (!ok) break;
#pragma unroll 1
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint64_t bh = sw128_mnmajor_desc(nh + ks * 2048, 0, 1024);
          const uint64_t bl = sw128_mnmajor_desc(nl + ks * 2048, 0, 1024);
          umma_bf16_ts_w(tmem + kTP, tmem + kTSH + ks * 8, bh, id_p, 1u);
          umma_bf16_ts_w(tmem + kTP, tmem + kTSH + ks * 8, bl, id_p, 1u);
          umma_bf16_ts_w(tmem + kTP, tmem + kTSL + ks * 8, bh, id_p, 1u);
        }
        umma_commit_w(p_full);
        // S += Y K: M = 128, N = d_k, K = 64 tokens; the key tile read as an MN-major B
        // (128-byte rows of 64 key columns per token, column blocks 8 KB apart, 8 tokens per 1 KB)
        ok = __all_sync(kFull, mbar_wait_bounded(y_full, c & 1));
        tc_fence_after();
        if (!ok) break;
#pragma unroll 1
        for (int ks = 0; ks < kC / 16; ++ks) {
          const uint64_t b = sw128_mnmajor_desc(kb + ks * 2048, 8192, 1024);
          umma_bf16_ts_w(tmem + kTS, tmem + kTYH + ks * 8, b, id_s, 1u);
          umma_bf16_ts_w(tmem + kTS, tmem + kTYL + ks * 8, b, id_s, 1u);
        }
        umma_commit_w(s_full);
        umma_commit_w(&empty[s]);
      }
      if (c + 1 < nch) ok = issue_u(c + 1);      // P's columns were read by the Y split (y_full)
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
    bool ok = convert_n(tl, sm + kOffN + uint32_t(i) * 128u, i, n_full, n_ready, 0);
    for (int c = 0; c < nch && ok; ++c) {
      const int s = c % kStages;
      ok = mbar_wait_bounded(p_full, c & 1);
      if (!__all_sync(kFull, ok)) break;
      tc_fence_after();
      // Y = P as bf16 hi + lo
#pragma unroll 1
      for (int q = 0; q < 2; ++q) {
        float x[32];
        tmem_ld32(tl + kTP + 32 * q, x);
        uint4 hi[4], lo[4];
        split32(x, hi, lo);
        tmem_st16(tl + kTYH + 16 * q, hi);
        tmem_st16(tl + kTYL + 16 * q, lo);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(y_full);
        mbar_arrive(&empty[s]);                      // done with this stage's scalars
      }
      const bool last = c + 1 == nch;
      const int s1 = (c + 1) % kStages;
      // the next chunk's N while S is updated, when it is already there
      bool converted = last;
      if (!last && __all_sync(kFull, mbar_test(n_full, (c + 1) & 1))) {
        if (!(ok = convert_n(tl, sm + kOffN + uint32_t(i) * 128u, i, n_full, n_ready, c + 1)))
          break;
        converted = true;
      }
      // the state leaving the chunk, in one pass: bf16 hi + lo for the next P, then a_C S for
      // the next accumulation
      ok = mbar_wait_bounded(s_full, c & 1);
      if (!last) ok = ok && mbar_wait_bounded(&pre[s1], ((c + 1) / kStages) & 1);
      if (!__all_sync(kFull, ok)) break;
      tc_fence_after();
      if (!last) {
        const float aC =
            reinterpret_cast<const float*>(sm + kOffSc + s1 * kScFloats * 4)[3 * kC];
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          float x[32];
          tmem_ld32(tl + kTS + 32 * q, x);
          uint4 hi[4], lo[4];
          split32(x, hi, lo);
          tmem_st16(tl + kTSH + 16 * q, hi);
          tmem_st16(tl + kTSL + 16 * q, lo);
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] *= aC;
          tmem_st32(tl + kTS + 32 * q, x);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(shl_full);
        if (!converted &&
            !(ok = convert_n(tl, sm + kOffN + uint32_t(i) * 128u, i, n_full, n_ready, c + 1)))
          break;
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
    // group grp takes chunks grp, grp + 2, ...; ptid = thread within the group, qd = the
    // warp's tensor-memory lane quarter
    const int grp = warp >= kWPre1 ? 1 : 0;
    const int ptid = tid - 32 * (grp ? kWPre1 : 0), pbar = kBarPre + grp;
    const int qd = warp & 3;
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
      const int s = c % kStages, n = c / kStages, cc = c >> 1;
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
      const float GC = Gs[kC - 1], aC = expf(GC);
      if (ptid < kC) {
        sc[ptid] = bcur;
        sc[kC + ptid] = bcur * expf(GC - G);
        sc[2 * kC + ptid] = -expf(G);
      }
      if (ptid == 0) sc[3 * kC] = aC;
      named_bar_sync(pbar, 128);
      // L = diag(beta) K~ from the Gram matrix in tensor memory, by the group's two warps on
      // lane quarters 0 and 1 (thread = token j; whole rows are written, but only the entries
      // below the diagonal are ever read). L shares its shared memory with M1 and T with M2: the U and N products of the
      // group's previous chunk have read them (m_free) before L is written.
      if (qd < 2) {
        ok = mbar_wait_bounded(&kk_full[grp], cc & 1) &&
             (cc == 0 || mbar_wait_bounded(&m_free[grp], (cc - 1) & 1));
        if (__all_sync(kFull, ok)) {
          tc_fence_after();
          const int j = 32 * qd + lane;
          float x0[32], x1[32];
          tmem_ld32(tmem + (uint32_t(32 * qd) << 16) + kTG, x0);
          tmem_ld32(tmem + (uint32_t(32 * qd) << 16) + kTG + 32, x1);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(kk_free);
          const float bjv = sc[j];
          float4* lrow = reinterpret_cast<float4*>(Lm + j * kLd);
#pragma unroll
          for (int m4 = 0; m4 < 8; ++m4) {
            lrow[m4] = make_float4(bjv * x0[4 * m4], bjv * x0[4 * m4 + 1], bjv * x0[4 * m4 + 2],
                                   bjv * x0[4 * m4 + 3]);
            lrow[8 + m4] = make_float4(bjv * x1[4 * m4], bjv * x1[4 * m4 + 1],
                                       bjv * x1[4 * m4 + 2], bjv * x1[4 * m4 + 3]);
          }
        } else {
          ok = false;
        }
      }
      if (!bar_and(pbar, 128, ok)) {
        if (ptid == 0) report_error(a.err, OLA_ERR_TIMEOUT, 44, c);
        break;
      }
      // T = (I + L)^-1: the four 16 x 16 diagonal blocks by forward substitution (thread =
      // column), then the blocks below them
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
      // The off-diagonal blocks as two halves of 32: T = [[A, 0], [C, B]] with A, B the inverses
      // of the two diagonal 32 x 32 parts and C = -B L_(23)(01) A. Each half's lower block
      // first (T_10 = -T_11 L_10 T_00, T_32 = -T_33 L_32 T_22), then X = L_(23)(01) A and
      // C = -B X; 16 x 16 block products, four barriers. Scratch (Qb): Y, then X.
      {
        // Y_h = L_(h+1)(h) T_hh for h = 0, 2 (thread = half, row y, 4 columns)
        const int hb = 2 * (ptid >> 6), y = (ptid >> 2) & 15, x0 = (ptid & 3) * 4;
        const float* lrow = Lm + (16 * hb + 16 + y) * kLd + 16 * hb;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int z = 0; z < 16; ++z) {
          const float l = lrow[z];
          const float4 t = *reinterpret_cast<const float4*>(Tf + (16 * hb + z) * kLdT + 16 * hb + x0);
          acc.x += l * t.x;
          acc.y += l * t.y;
          acc.z += l * t.z;
          acc.w += l * t.w;
        }
        *reinterpret_cast<float4*>(Qb + (hb / 2) * 256 + y * 16 + x0) = acc;
        named_bar_sync(pbar, 128);
        // T_(h+1)(h) = -T_(h+1)(h+1) Y_h
        const float* trow = Tf + (16 * hb + 16 + y) * kLdT + 16 * hb + 16;
        float4 t2 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int z = 0; z < 16; ++z) {
          const float tz = trow[z];
          const float4 q = *reinterpret_cast<const float4*>(Qb + (hb / 2) * 256 + z * 16 + x0);
          t2.x -= tz * q.x;
          t2.y -= tz * q.y;
          t2.z -= tz * q.z;
          t2.w -= tz * q.w;
        }
        *reinterpret_cast<float4*>(Tf + (16 * hb + 16 + y) * kLdT + 16 * hb + x0) = t2;
        named_bar_sync(pbar, 128);
      }
      {
        // X_(br)(bc) = sum_{kb = bc..1} L_(br)(kb) T_(kb)(bc), br in {2, 3}, bc in {0, 1}
        // (thread = block, rows 2 rp and 2 rp + 1, 4 columns); then C = -B X
        const int blk = ptid >> 5, br = 2 + (blk >> 1), bc = blk & 1;
        const int rp = (ptid >> 2) & 7, x0 = (ptid & 3) * 4;
        const float* l0 = Lm + (16 * br + 2 * rp) * kLd;
        const float* l1 = l0 + kLd;
        float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
#pragma unroll 1
        for (int kb = bc; kb < 2; ++kb) {
#pragma unroll 4
          for (int z = 0; z < 16; ++z) {
            const float u0 = l0[16 * kb + z], u1 = l1[16 * kb + z];
            const float4 t =
                *reinterpret_cast<const float4*>(Tf + (16 * kb + z) * kLdT + 16 * bc + x0);
            a0.x += u0 * t.x;
            a0.y += u0 * t.y;
            a0.z += u0 * t.z;
            a0.w += u0 * t.w;
            a1.x += u1 * t.x;
            a1.y += u1 * t.y;
            a1.z += u1 * t.z;
            a1.w += u1 * t.w;
          }
        }
        float* xb = Qb + blk * 256;                     // X_(br)(bc) at ((br - 2) * 2 + bc)
        *reinterpret_cast<float4*>(xb + (2 * rp) * 16 + x0) = a0;
        *reinterpret_cast<float4*>(xb + (2 * rp + 1) * 16 + x0) = a1;
        named_bar_sync(pbar, 128);
        // C_(br)(bc) = -sum_{kb = 2..br} T_(br)(kb) X_(kb)(bc)
        const float* t0 = Tf + (16 * br + 2 * rp) * kLdT;
        const float* t1 = t0 + kLdT;
        float4 c0 = make_float4(0.f, 0.f, 0.f, 0.f), c1 = c0;
#pragma unroll 1
        for (int kb = 2; kb <= br; ++kb) {
          const float* xk = Qb + ((kb - 2) * 2 + bc) * 256;
#pragma unroll 4
          for (int z = 0; z < 16; ++z) {
            const float u0 = t0[16 * kb + z], u1 = t1[16 * kb + z];
            const float4 q = *reinterpret_cast<const float4*>(xk + z * 16 + x0);
            c0.x -= u0 * q.x;
            c0.y -= u0 * q.y;
            c0.z -= u0 * q.z;
            c0.w -= u0 * q.w;
            c1.x -= u1 * q.x;
            c1.y -= u1 * q.y;
            c1.z -= u1 * q.z;
            c1.w -= u1 * q.w;
          }
        }
        *reinterpret_cast<float4*>(Tf + (16 * br + 2 * rp) * kLdT + 16 * bc + x0) = c0;
        *reinterpret_cast<float4*>(Tf + (16 * br + 2 * rp + 1) * kLdT + 16 * bc + x0) = c1;
        named_bar_sync(pbar, 128);
      }
      // M1 (over L), then M2 (over T) as bf16 hi and lo, K-major tiles with the 128-byte
      // swizzle: tile row = output token (the N index), column = source token j (the K index);
      // thread = half a row, 16 bytes (8 columns) at a time. M2_jm = M1_jm (-a_j), formed from
      // M1's hi + lo once every T entry has been read.
      {
        const int jr = ptid >> 1, hf = ptid & 1;
        unsigned char* m1h = gb + kGL;
        unsigned char* m2h = gb + kGTf;
#pragma unroll 1
        for (int qq = 0; qq < 4; ++qq) {
          const int q = 4 * hf + qq, m0 = 8 * q;
          const float4 t0 = *reinterpret_cast<const float4*>(Tf + jr * kLdT + m0);
          const float4 t1 = *reinterpret_cast<const float4*>(Tf + jr * kLdT + m0 + 4);
          const float4 b0 = *reinterpret_cast<const float4*>(sc + kC + m0);
          const float4 b1 = *reinterpret_cast<const float4*>(sc + kC + m0 + 4);
          // entries past the diagonal are not T's (zero, or stale in blocks above it)
          const float t[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
          const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            split2(m0 + 2 * e <= jr ? t[2 * e] * b[2 * e] : 0.f,
                   m0 + 2 * e + 1 <= jr ? t[2 * e + 1] * b[2 * e + 1] : 0.f, hw[e], lw[e]);
          const uint32_t off = uint32_t(jr) * 128u + uint32_t((q ^ (jr & 7)) << 4);
          *reinterpret_cast<uint4*>(m1h + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(m1h + kMTile + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        named_bar_sync(pbar, 128);
#pragma unroll 1
        for (int qq = 0; qq < 4; ++qq) {
          const int q = 4 * hf + qq, m0 = 8 * q;
          const uint32_t off = uint32_t(jr) * 128u + uint32_t((q ^ (jr & 7)) << 4);
          const uint4 h = *reinterpret_cast<const uint4*>(m1h + off);
          const uint4 l = *reinterpret_cast<const uint4*>(m1h + kMTile + off);
          const float4 a0 = *reinterpret_cast<const float4*>(sc + 2 * kC + m0);
          const float4 a1 = *reinterpret_cast<const float4*>(sc + 2 * kC + m0 + 4);
          const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, lw[4] = {l.x, l.y, l.z, l.w};
          const float na[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
          uint32_t h2[4], l2[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // bf16 pairs back to fp32: the low half holds the first column
            const float x0 = __uint_as_float(hw[e] << 16) + __uint_as_float(lw[e] << 16);
            const float x1 =
                __uint_as_float(hw[e] & 0xffff0000u) + __uint_as_float(lw[e] & 0xffff0000u);
            split2(x0 * na[2 * e], x1 * na[2 * e + 1], h2[e], l2[e]);
          }
          *reinterpret_cast<uint4*>(m2h + off) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
          *reinterpret_cast<uint4*>(m2h + kMTile + off) = make_uint4(l2[0], l2[1], l2[2], l2[3]);
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
// one 64-column block of 64 consecutive tokens of one (request, head), stored with the 128-byte
// swizzle (the tensor cores read it K-major and MN-major). Tokens past P read 0.
bool make_prompt_map(CUtensorMap* map, const void* base, int R, int P, int H) {
  EncodeFn fn = prompt_encoder();
  if (!fn) return false;
  cuuint64_t dims[4] = {cuuint64_t(kD), cuuint64_t(H), cuuint64_t(P), cuuint64_t(R)};
  cuuint64_t strides[3] = {cuuint64_t(kD) * 2, cuuint64_t(H) * kD * 2,
                           cuuint64_t(P) * H * kD * 2};
  cuuint32_t box[4] = {64, 1, kC, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B,
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
  if (!make_prompt_map(&a.mk, k, R, P, H) || !make_prompt_map(&a.mv, v, R, P, H))
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
