// la_gdn.cu -- the gated delta rule in chunks, on the sm_100a tensor cores
// (tcgen05 + TMA + TMEM), bf16 inputs, fp32 accumulation and state.
//
// The rule ("1.6 长上下文与高效注意力", section Gated delta rule): with unit keys
// kt_t = k_t / max(|k_t|, 1e-12) and alpha_t = exp(g_t),
//     S_t = alpha_t S_{t-1} (I - beta_t kt_t kt_t^T) + beta_t v_t kt_t^T,   o_t = S_t q_t.
// Regrouped over a chunk of C tokens that starts from state S_0 (b_i = the sum
// of g over the chunk's tokens 0..i), token i writes u_i kt_i^T with
// u_i = beta_i (v_i - alpha_i S_{i-1} kt_i), so
//     S_i = e^{b_i} S_0 + sum_{j<=i} e^{b_i - b_j} u_j kt_j^T.
// Putting that S_{i-1} into u_i makes the rows u_i the solution of a unit
// lower-triangular system.  With A_ij = beta_i e^{b_i - b_j} (kt_i . kt_j) for
// j < i and T = (I + A)^{-1} (the "UT transform" of the chunk):
//     U  = Ut - W S_0^T,     Ut = T diag(beta) V,     W = T diag(beta e^b) Kt,
//     O  = diag(e^b) Q S_0^T + (tril(Q Kt^T) .* D) U,      D_ij = e^{b_i - b_j},
//     S' = e^{b_last} S_0 + (diag(e^{b_last - b}) Kt)^T U.
// Ut and W depend on the chunk's own inputs only; U, O and S' need the state.
// Two kernels:
//   gdn_prep_kernel  one CTA per (sequence, chunk, head), all independent: G =
//                    K K^T on the tensor cores; A from G and the key norms; T
//                    by forward substitution on the CUDA cores (fp32); then
//                    W = T diag(beta e^b) Kt and Ut = T diag(beta) V on the
//                    tensor cores.  W and Ut go to the workspace as bf16
//                    [B, T, H, 128], with the chunk's b_i and ln(1/|k_i|) - b_i.
//   gdn_tc_kernel    one CTA per (sequence, head) walks its chunks in order with
//                    the fp32 state S^T in registers, as the linear-attention
//                    forward does.  Per chunk, five products:
//                      MW  WS = W Sb                 (M=C, N=d_v, K=d_k)   Sb = bf16(S^T)
//                      M1  A  = Q K^T                (M=C, N=C,   K=d_k)   raw keys
//                      M4  Us = Kd^T U               (M=d_k, N=d_v, K=C)   Kd = diag(e^{b_last-b}) Kt
//                      M2  O  = Qd Sb                (M=C, N=d_v, K=d_k)   Qd = diag(e^b) Q
//                      M3  O += P U                  (M=C, N=d_v, K=C)     P_ij = A_ij D_ij / |k_j|, j <= i
//                    with U = Ut - WS between MW and M4 and S^T <- e^{b_last} S^T + Us after M4.
//                    The key norms enter through the table c_j = ln(1/|k_j|) - b_j: P's
//                    factor is e^{b_i + c_j}, Kd's row factor e^{b_last + c_j}.
//   Warp roles of gdn_tc_kernel (384 threads, as in the forward):
//     warp 0      TMA producer: Q, K, W, Ut chunk tiles and the chunk's table into a two-deep ring.
//     warp 1      TMEM allocator and single-thread tcgen05.mma issuer.
//     warps 2-3   transform: the decayed unit keys Kd.
//     warps 4-7   state: S^T update, the bf16 operand Sb, and U = Ut - WS in place.
//     warps 8-11  output: score tile -> P, Qd in place, epilogue.
// Every wait is bounded: on a timeout the CTA raises an abort flag, records the
// failure in a device error word, drains and frees its tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_common.cuh"
#include "la_internal.h"
#include "la_sm100.cuh"
#include "la_tc_sync.cuh"

namespace la {

__device__ unsigned int g_gdn_error = 0;
// First wait that gave up: 0x80000000 | chunk << 8 | barrier index.
__device__ unsigned int g_gdn_where = 0;

namespace {

using namespace sm100;
using namespace tcsync;

constexpr int kC = 64;            // chunk length
constexpr int kD = 128;           // d_k = d_v on this path
constexpr int kSlab = kC * 128;   // one [C rows x 64 cols] bf16 slab, 128-byte swizzled
constexpr int kTile = 2 * kSlab;  // one [C x 128] tile

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
  return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Byte offset of the 16-byte chunk holding logical columns [8p, 8p + 8) of row r
// in a 128-byte-swizzled [rows x 64] slab.
__device__ __forceinline__ int swz(int r, int p) { return r * 128 + ((p ^ (r & 7)) << 4); }

// Start-address offset (16-byte units) of K step kk (16 columns) in a K-major
// operand made of 64-column slabs.
__device__ __forceinline__ uint32_t kmaj(int kk) { return (uint32_t)(((kk >> 2) * kSlab + (kk & 3) * 32) >> 4); }

// Sequence, first token and length of sequence n: dense batches hold B
// sequences of T tokens; packed ones one row of sequences cut by cu_seqlens.
struct SeqPos {
  int64_t bidx, start, len;
};
__device__ __forceinline__ SeqPos seq_pos(const int32_t *cu, int64_t n, int64_t T) {
  if (cu) return SeqPos{0, (int64_t)cu[n], (int64_t)cu[n + 1] - cu[n]};
  return SeqPos{n, 0, T};
}

// ============================================================== prep kernel
struct PrepArgs {
  const float *g, *beta;      // [B * T][H]
  const int32_t *cu_seqlens;  // NULL: dense
  const int32_t *coff;        // packed: first chunk slot of each sequence, [n_seqs + 1]
  __nv_bfloat16 *w, *ut;  // [B, T, H, 128] each: W and T diag(beta) V
  float *bt;               // [chunk slot][H][2][C]: b_i (rows past the chunk end repeat b_last), then
                           // c_i = ln(1/|k_i|) - b_i (-inf there)
  int64_t T, n_seqs;
  int H;
  int skip_load;  // testing the failure path: no tile load, so the first wait runs out
};

struct PrepCfg {
  static constexpr int OFF_K = 0;              // K (rows past the chunk end zeroed)
  static constexpr int OFF_V = OFF_K + kTile;  // V (likewise)
  // A, fp32 [C][A_LD], inverted in place; then T diag(beta) and T diag(beta e^b / |k|), bf16
  static constexpr int OFF_A = OFF_V + kTile;
  static constexpr int A_LD = kC + 4;          // rows 16-byte aligned for float4 access
  static constexpr int OFF_VEC = OFF_A + kC * A_LD * 4;  // b_i, beta_i, 1/max(|k_i|, 1e-12): 3 x C floats
  static constexpr int OFF_BAR = OFF_VEC + 3 * kC * 4;   // 0: tiles landed, 1: products done
  static constexpr int OFF_MISC = OFF_BAR + 2 * 8;
  static constexpr int SMEM_USED = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
  static constexpr int T_COLS = 128;                   // four CTAs per SM fill the tensor memory
  static_assert(4 * (SMEM_BYTES + 1024) <= 233472, "four prep CTAs per SM");
  static_assert(5 * (SMEM_BYTES + 1024) > 233472, "at most four prep CTAs per SM (tensor memory)");
  static_assert(OFF_A % 1024 == 0, "T^T tile alignment");
};

// Sequence start slots of a packed batch: coff[n] = sum_{m<n} ceil(len_m / C).
// One block; the counts are scanned 1024 sequences at a time.
__global__ void __launch_bounds__(1024) gdn_chunk_offsets_kernel(const int32_t *cu, int64_t n_seqs,
                                                                 int32_t *coff) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    carry = 0;
    coff[0] = 0;
  }
  __syncthreads();
  for (int64_t base = 0; base < n_seqs; base += 1024) {
    const int64_t n = base + tid;
    int32_t x = n < n_seqs ? (int32_t)(((int64_t)cu[n + 1] - cu[n] + kC - 1) / kC) : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int32_t s = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      warp_sums[lane] = s;
    }
    __syncthreads();
    const int32_t incl = x + (warp > 0 ? warp_sums[warp - 1] : 0) + carry;
    if (n < n_seqs) coff[n + 1] = incl;
    __syncthreads();
    if (tid == 1023) carry = incl;
    __syncthreads();
  }
}

// ---- T = (I + A)^{-1} for the strictly lower-triangular C x C matrix A (fp32,
// leading dimension A_LD), in place, by blocks.  With L = I + A split into
// halves, L = [L1 0; L21 L2] gives L^{-1} = [L1^{-1} 0; -L2^{-1} L21 L1^{-1} L2^{-1}],
// and the same split of each 32 x 32 half into 16 x 16 blocks D_k = (I + A_kk)^{-1}:
//   level 0  the four D_k by forward substitution in fp32 (thread = one column of one block)
//   level 1  the lower-left 16 x 16 block of each half, -D_1 A_10 D_0 and -D_3 A_32 D_2
//   level 2  the lower-left 32 x 32 block, -L2^{-1} (L21 L1^{-1})
// The block products run on the warp-level tensor-core instruction (mma.sync
// m16n8k8, tf32 inputs rounded to nearest, fp32 accumulation): 16 x 8 tiles,
// with operands loaded straight from the fp32 matrix (conflict-free at this
// leading dimension).  Intermediate blocks use the (zero) upper triangle.

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// d = X[16 rows][K] Y[K][8 cols] for one warp (X, Y fp32, leading dimension A_LD).  Lane
// l holds rows l / 4 and l / 4 + 8, columns 2 (l % 4) and 2 (l % 4) + 1.
template <int K>
__device__ __forceinline__ void tile_product(const float *X, const float *Y, int lane, float (&d)[4]) {
  constexpr int LD = PrepCfg::A_LD;
  const int g = lane >> 2, t = lane & 3;
  d[0] = d[1] = d[2] = d[3] = 0.f;
#pragma unroll
  for (int k0 = 0; k0 < K; k0 += 8) {
    const uint32_t a0 = to_tf32(X[g * LD + k0 + t]), a1 = to_tf32(X[(g + 8) * LD + k0 + t]);
    const uint32_t a2 = to_tf32(X[g * LD + k0 + t + 4]), a3 = to_tf32(X[(g + 8) * LD + k0 + t + 4]);
    const uint32_t b0 = to_tf32(Y[(k0 + t) * LD + g]), b1 = to_tf32(Y[(k0 + t + 4) * LD + g]);
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ void store_tile(float *dst, const float (&d)[4], int lane, float sc) {
  constexpr int LD = PrepCfg::A_LD;
  const int g = lane >> 2, t = lane & 3;
  *reinterpret_cast<float2 *>(dst + g * LD + 2 * t) = make_float2(sc * d[0], sc * d[1]);
  *reinterpret_cast<float2 *>(dst + (g + 8) * LD + 2 * t) = make_float2(sc * d[2], sc * d[3]);
}

// Called by all 128 threads of the CTA (contains __syncthreads).
__device__ __forceinline__ void invert_unit_lower(float *As, int tid) {
  constexpr int LD = PrepCfg::A_LD;
  const int warp = tid >> 5, lane = tid & 31;
  // level 0: thread tid < 64 solves column j of block k: x_i = [i == j] - sum_{m<i} A_kk[i][m] x_m
  float x[16];
  const int k0 = tid >> 4, j0 = tid & 15;
  if (tid < 64) {
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float *arow = As + (16 * k0 + i) * LD + 16 * k0;
      float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int m = 0; m < i; m += 4) {  // A_im = 0 for m >= i; x_m = 0 beyond what is solved
        const float4 av = *reinterpret_cast<const float4 *>(arow + m);
        s0 = __ffma2_rn(make_float2(av.x, av.y), make_float2(x[m], x[m + 1]), s0);
        s1 = __ffma2_rn(make_float2(av.z, av.w), make_float2(x[m + 2], x[m + 3]), s1);
      }
      x[i] = i < j0 ? 0.f : (i == j0 ? 1.f : -((s0.x + s0.y) + (s1.x + s1.y)));
    }
  }
  __syncthreads();  // the diagonal blocks of A are read: D_k replaces them
  if (tid < 64) {
#pragma unroll
    for (int i = 0; i < 16; ++i) As[(16 * k0 + i) * LD + 16 * k0 + j0] = x[i];
  }
  __syncthreads();
  // level 1: warp 0 the first half (blocks 0, 1), warp 1 the second (blocks 2, 3)
  if (warp < 2) {
    const int o = 32 * warp;
    float d[2][4];
    // X = A_10 D_0 into the (zero) upper block (0, 1) of the half
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) tile_product<16>(As + (o + 16) * LD + o, As + o * LD + o + 8 * nt, lane, d[nt]);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) store_tile(As + o * LD + o + 16 + 8 * nt, d[nt], lane, 1.f);
    __syncwarp();
    // -D_1 X over A_10
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
      tile_product<16>(As + (o + 16) * LD + o + 16, As + o * LD + o + 16 + 8 * nt, lane, d[nt]);
    __syncwarp();
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) store_tile(As + (o + 16) * LD + o + 8 * nt, d[nt], lane, -1.f);
    // the scratch block back to zero
    const float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) store_tile(As + o * LD + o + 16 + 8 * nt, z, lane, 1.f);
  }
  __syncthreads();
  // level 2: Y = L21 L1^{-1} (32 x 32) into the upper-right quarter, then -L2^{-1} Y over L21;
  // warp w: row tile w % 2, column tiles 2 (w / 2) and 2 (w / 2) + 1
  {
    const int mt = warp & 1, n0 = 2 * (warp >> 1);
    float d[2][4];
#pragma unroll
    for (int u = 0; u < 2; ++u) tile_product<32>(As + (32 + 16 * mt) * LD, As + 8 * (n0 + u), lane, d[u]);
#pragma unroll
    for (int u = 0; u < 2; ++u) store_tile(As + 16 * mt * LD + 32 + 8 * (n0 + u), d[u], lane, 1.f);
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 2; ++u)
      tile_product<32>(As + (32 + 16 * mt) * LD + 32, As + 32 + 8 * (n0 + u), lane, d[u]);
#pragma unroll
    for (int u = 0; u < 2; ++u) store_tile(As + (32 + 16 * mt) * LD + 8 * (n0 + u), d[u], lane, -1.f);
  }
  __syncthreads();
}

// One CTA per (sequence, chunk, head), four per SM.  Thread tt owns the
// 16-byte vectors tt + 128 m (m < 8) of a [C x 128] tile: rows tt/8 + 16 m'
// (m' < 4) in both 64-column slabs, physical chunk tt mod 8; the 8 lanes of a
// row differ in their low three bits.
__global__ void __launch_bounds__(128, 4) gdn_prep_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                          const __grid_constant__ CUtensorMap tm_v,
                                                          const PrepArgs a) {
  using P = PrepCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = align1024(smem_raw);
  float *As = reinterpret_cast<float *>(sm + P::OFF_A);
  float *bvec = reinterpret_cast<float *>(sm + P::OFF_VEC);
  float *betav = bvec + kC;
  float *invn = betav + kC;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + P::OFF_BAR);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + P::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + P::OFF_MISC + 4);
  const Sync sy{bars, abort_flag, &g_gdn_error, &g_gdn_where};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- this CTA's (sequence, chunk, head); heads vary fastest
  const int h = (int)(blockIdx.x % a.H);
  const int64_t slot = blockIdx.x / a.H;
  int64_t n, c;
  if (a.coff) {
    if (slot >= a.coff[a.n_seqs]) return;  // past the last chunk (the grid is an upper bound)
    int64_t lo = 0, hi = a.n_seqs - 1;     // last n with coff[n] <= slot: never an empty sequence
    while (lo < hi) {
      const int64_t mid = (lo + hi + 1) >> 1;
      if (a.coff[mid] <= slot)
        lo = mid;
      else
        hi = mid - 1;
    }
    n = lo;
    c = slot - a.coff[n];
  } else {
    const int64_t nck = (a.T + kC - 1) / kC;
    n = slot / nck;
    c = slot % nck;
  }
  const SeqPos sp = seq_pos(a.cu_seqlens, n, a.T);
  const int64_t t0 = sp.start + c * kC;  // first token of the chunk in its batch row
  const int Cp = (int)min((int64_t)kC, sp.len - c * kC);

  // ---- setup: barriers, tensor memory, the tile loads, b_i and beta_i
  if (tid == 0) {
    mbar_init(bars + 0, 1);
    mbar_init(bars + 1, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (!a.skip_load) {
      mbar_arrive_expect_tx(bars + 0, 2 * kTile);
      for (int kb = 0; kb < 2; ++kb) {
        tma_load_4d(sm + P::OFF_K + kb * kSlab, &tm_k, bars + 0, kb * 64, h, (int)t0, (int)sp.bidx);
        tma_load_4d(sm + P::OFF_V + kb * kSlab, &tm_v, bars + 0, kb * 64, h, (int)t0, (int)sp.bidx);
      }
    }
  }
  // Give up the allocation permit at once: an SM takes no further CTA while one
  // of its CTAs still holds the permit (measured), and four CTAs fill the tensor memory.
  if (warp == 1) {
    tmem_alloc(tmem_slot, P::T_COLS);
    tmem_relinquish();
  }
  if (warp == 0) {  // b_i = sum_{t<=i} g_t over the chunk (rows past its end add 0 and get beta = 0)
    const int64_t row0 = (sp.bidx * a.T + t0) * a.H + h;
    float blo = lane < Cp ? a.g[row0 + (int64_t)lane * a.H] : 0.f;
    float bhi = lane + 32 < Cp ? a.g[row0 + (int64_t)(lane + 32) * a.H] : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y0 = __shfl_up_sync(0xffffffffu, blo, o);
      const float y1 = __shfl_up_sync(0xffffffffu, bhi, o);
      if (lane >= o) {
        blo += y0;
        bhi += y1;
      }
    }
    bhi += __shfl_sync(0xffffffffu, blo, 31);
    bvec[lane] = blo;
    bvec[lane + 32] = bhi;
    float *btab = a.bt + (slot * a.H + h) * 2 * kC;
    btab[lane] = blo;
    btab[lane + 32] = bhi;
    betav[lane] = lane < Cp ? a.beta[row0 + (int64_t)lane * a.H] : 0.f;
    betav[lane + 32] = lane + 32 < Cp ? a.beta[row0 + (int64_t)(lane + 32) * a.H] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  bool ok = wait_bar_warp(sy, 0, 0);
  int issued = 0;  // products committed on barrier 1 (thread 0)

  // G = K K^T from the raw keys (M = N = C, K = 128) into columns [0, C); the
  // norms are applied to G afterwards
  if (ok && tid == 0) {
    tc_fence_after();
    const uint64_t dk = smem_desc_sw128(smem_u32(sm + P::OFF_K), 16, 1024);
    constexpr uint32_t ID_G = idesc_bf16_f32(kC, kC, 0, 0);
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) umma_bf16(tbase, dk + kmaj(kk), dk + kmaj(kk), ID_G, kk > 0);
    umma_commit(bars + 1);
    issued = 1;
  }
  // while it runs: 1/|k_i|.  Rows past the chunk end must not reach the products below
  // (they may hold anything): V rows become zero here, K rows once G is done.
  if (ok) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int r = (tid >> 3) + 16 * m;
      const int off = (tid + 128 * m) * 16;
      float f0[8], f1[8];
      unpack8(*reinterpret_cast<const uint4 *>(sm + P::OFF_K + off), f0);
      unpack8(*reinterpret_cast<const uint4 *>(sm + P::OFF_K + kSlab + off), f1);
      float ss = 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) ss = fmaf(f0[u], f0[u], fmaf(f1[u], f1[u], ss));
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      ss += __shfl_xor_sync(0xffffffffu, ss, 4);
      if ((tid & 7) == 0) invn[r] = r < Cp ? 1.f / fmaxf(sqrtf(ss), 1e-12f) : 0.f;
      if (r >= Cp) {
        *reinterpret_cast<uint4 *>(sm + P::OFF_V + off) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4 *>(sm + P::OFF_V + kSlab + off) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  __syncthreads();  // 1/|k| of every row
  // for the chunk kernel: e^{b_i + c_j} = e^{b_i - b_j} / |k_j|, one exponential per factor
  if (tid < kC) a.bt[(slot * a.H + h) * 2 * kC + kC + tid] = __logf(invn[tid]) - bvec[tid];
  ok = ok && wait_bar_warp(sy, 1, 0);
  tc_fence_after();
  if (ok) {
    // A_ij = beta_i e^{b_i - b_j} kt_i . kt_j for j < i < C': row i, 32 columns
    const int i = (warp & 3) * 16 + (lane & 15), hf = lane >> 4;
    uint32_t r[32];
    tmem_ld_16x32bx2_x32<32>(tbase + ((uint32_t)(warp * 32) << 16), r);
    tmem_wait_ld();
    const float bi = bvec[i], wi = i < Cp ? betav[i] * invn[i] : 0.f;
    float4 *arow = reinterpret_cast<float4 *>(As + i * P::A_LD + hf * 32);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float e4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = hf * 32 + 4 * q + u;
        e4[u] = (j < i && i < Cp) ? wi * invn[j] * exp_fast(bi - bvec[j]) * __uint_as_float(r[4 * q + u]) : 0.f;
      }
      arow[q] = make_float4(e4[0], e4[1], e4[2], e4[3]);
    }
    // K rows past the chunk end to zero (the product has read K)
    if (Cp < kC) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        if ((tid >> 3) + 16 * m < Cp) continue;
        *reinterpret_cast<uint4 *>(sm + P::OFF_K + (tid + 128 * m) * 16) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4 *>(sm + P::OFF_K + kSlab + (tid + 128 * m) * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  // ---- T = (I + A)^{-1} in place (fp32).  The row scalings of the right-hand sides
  // move onto the columns of T: W = (T diag(beta e^b / |k|)) K and Ut = (T diag(beta)) V,
  // stored as two bf16 [C x C] tiles in the MN-major layout (row j = column j of T).
  // Thread (j, hr) handles rows [32 hr, 32 hr + 32) of column j.
  // (every thread takes part, whatever `ok` says: the inverse synchronises the CTA)
  invert_unit_lower(As, tid);
  {
    const int j = tid & 63, hr = tid >> 6;
    const float cu = betav[j], cw = cu * exp_fast(bvec[j]) * invn[j];
    float tc[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int i = 32 * hr + u;  // zero above the diagonal (the upper triangle held scratch)
      tc[u] = i >= j ? As[i * P::A_LD + j] : 0.f;
    }
    __syncthreads();
    uint8_t *tu = sm + P::OFF_A, *tw = sm + P::OFF_A + kSlab;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float fu[8], fw[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        fu[u] = tc[8 * q + u] * cu;
        fw[u] = tc[8 * q + u] * cw;
      }
      *reinterpret_cast<uint4 *>(tu + swz(j, 4 * hr + q)) = pack8(fu);
      *reinterpret_cast<uint4 *>(tw + swz(j, 4 * hr + q)) = pack8(fw);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  // ---- W, then Ut (M = C, N = 128, K = C), each into columns [0, 128) and stored as bf16
  // rows of the workspace
  constexpr uint32_t ID_X = idesc_bf16_f32(kC, kD, 1, 1);  // A = T-tile, MN-major
  const int i = (warp & 3) * 16 + (lane & 15), hf = lane >> 4;  // row and 64-column half read back
#pragma unroll 1
  for (int part = 0; part < 2; ++part) {
    if (ok && tid == 0) {
      tc_fence_after();
      const uint64_t dx = smem_desc_sw128(smem_u32(sm + (part ? P::OFF_V : P::OFF_K)), kSlab, 1024);
      const uint64_t dt = smem_desc_sw128(smem_u32(sm + P::OFF_A + (part ? 0 : kSlab)), kSlab, 1024);
#pragma unroll
      for (int kk = 0; kk < kC / 16; ++kk)
        umma_bf16(tbase, dt + ((kk * 2048) >> 4), dx + ((kk * 2048) >> 4), ID_X, kk > 0);
      umma_commit(bars + 1);
      issued = 2 + part;
    }
    ok = ok && wait_bar_warp(sy, 1, (part + 1) & 1);
    tc_fence_after();
    if (ok) {
      __nv_bfloat16 *dst = (part ? a.ut : a.w) + ((sp.bidx * a.T + t0 + i) * a.H + h) * (int64_t)kD + hf * 64;
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        uint32_t r[32];
        tmem_ld_16x32bx2_x32<64>(tbase + ((uint32_t)(warp * 32) << 16) + pass * 32, r);
        tmem_wait_ld();
        if (i < Cp) {
          uint4 *d4 = reinterpret_cast<uint4 *>(dst + pass * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            d4[q] = make_uint4(pack2(__uint_as_float(r[8 * q]), __uint_as_float(r[8 * q + 1])),
                               pack2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3])),
                               pack2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5])),
                               pack2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7])));
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // the columns are read before the next product overwrites them
  }
  // ---- teardown (after an abort, let the tile loads and products finish first)
  if (*abort_flag && tid == 0) {
    drain_bar(sy, 0, 0);
    for (int u = 0; u < issued; ++u) drain_bar(sy, 1, u & 1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, P::T_COLS);
}

// ============================================================== chunk kernel
constexpr int kThreads = 384;

struct GdnTcArgs {
  void *out;
  int64_t o_sb, o_st, o_sh;
  const float *bt;            // [chunk slot][H][2][C]: b_i and ln(1/|k_i|) - b_i of every chunk, from the WY pass
  const int32_t *coff;        // packed: first chunk slot of each sequence (dense: n * nck)
  int64_t nck;                // chunks per sequence (dense)
  const float *init;          // NULL or [n_seqs, H, d_k, d_v] (S^T)
  float *final_state;         // NULL or [n_seqs, H, d_k, d_v]
  const int32_t *cu_seqlens;  // NULL: dense
  int64_t T;
  int H;
  // head dims: 64 or 128 each; a 64 runs in the 128 layout, its extra key, query and
  // value columns read as TMA zero fill (zero rows and columns of S), never written out
  int dk, dv;
};

template <int NS>
struct GdnCfg {
  // a stage: Q (then Qd), K, W, Ut (then U), Kd; [C x 128] bf16 tiles
  static constexpr int OFF_Q = 0, OFF_K = kTile, OFF_W = 2 * kTile, OFF_U = 3 * kTile, OFF_KD = 4 * kTile;
  static constexpr int STAGE_BYTES = 5 * kTile;
  static constexpr int LOAD_BYTES = 4 * kTile + 2 * kC * 4;  // Q, K, W, Ut and the chunk's table arrive by TMA
  static constexpr int SB_SLAB = kD * 128;      // [d_k rows x 64 cols] bf16
  static constexpr int OFF_SB = NS * STAGE_BYTES;
  static constexpr int OFF_P = OFF_SB + 2 * SB_SLAB;
  static constexpr int OFF_DT = OFF_P + 2 * kSlab;  // per stage: b_i, then c_i (i < C); b_last = b_{C-1}
  static constexpr int DT_STRIDE = 2 * kC;
  static constexpr int OFF_BAR = OFF_DT + NS * DT_STRIDE * 4;
  static constexpr int B_FULL = 0, B_EMPTY = NS, B_XFORM = 2 * NS, B_QREADY = 3 * NS, B_AFULL = 4 * NS,
                       B_PFULL = 4 * NS + 2, B_OFULL = 4 * NS + 4, B_OEMPTY = 4 * NS + 6, B_WSFULL = 4 * NS + 8,
                       B_UREADY = 4 * NS + 9, B_UFULL = 4 * NS + 10, B_SBFULL = 4 * NS + 11,
                       B_SBEMPTY = 4 * NS + 12, NBAR = 4 * NS + 13;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_USED = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
  // tensor memory: Us / WS (time-shared), two score tiles, two output tiles
  static constexpr int T_U = 0, T_A = 128, T_O = 256, T_COLS = 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(OFF_BAR % 8 == 0, "barrier alignment");
};

// Thread roles and per-chunk protocol (chunk c, stage s = c % NS, b = c & 1;
// "prev" = the chunk starts from a state: c > 0 or an initial state):
//   MMA:       [prev: FULL, SBFULL] MW -> WSFULL;  [UREADY] M4 -> UFULL;
//              [OEMPTY[b], QREADY[s]] prev: M2 -> SBEMPTY;  [PFULL[b]] M3 -> OFULL[b], EMPTY[s];
//              [FULL(c+1)] M1 of chunk c + 1 -> AFULL[b ^ 1], issued between MW and M4 when
//              the tiles are in by then, else after M3 (M1 of chunk 0 before the loop).
//   state:     [UFULL(c-1)] S^T <- e^{b_last} S^T + Us;  [prev: SBEMPTY(c-1)] Sb -> SBFULL;
//              [XFORM, prev: WSFULL] U = Ut - WS in place -> UREADY.
//   output:    [AFULL[b], FULL] P -> PFULL[b];  Qd in place -> QREADY[s];
//              [OFULL[b-1]] epilogue of chunk c-1 -> OEMPTY.
//   transform: [FULL] Kd -> XFORM.
template <int NS>
__global__ void __launch_bounds__(kThreads, 1)
gdn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_u,
              const GdnTcArgs a) {
  using G = GdnCfg<NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = align1024(smem_raw);
  float *dtab = reinterpret_cast<float *>(sm + G::OFF_DT);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + G::OFF_BAR);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + G::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + G::OFF_MISC + 4);
  const Sync sy{bars, abort_flag, &g_gdn_error, &g_gdn_where};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int h = (int)(blockIdx.x % a.H);
  const int64_t n = blockIdx.x / a.H;
  const SeqPos sq = seq_pos(a.cu_seqlens, n, a.T);
  const int nchunks = (int)((sq.len + kC - 1) / kC);
  const bool has_init = a.init != nullptr;
  auto chunk_len = [&](int c) -> int { return (int)min((int64_t)kC, sq.len - (int64_t)c * kC); };
  auto prev = [&](int c) -> bool { return c > 0 || has_init; };
  // index of chunk c among the chunks that start from a state (parity of SBFULL, WSFULL, SBEMPTY)
  auto sbi = [&](int c) -> int { return c - 1 + (has_init ? 1 : 0); };
  auto stage = [&](int s) { return sm + s * G::STAGE_BYTES; };

  if (tid == 0) {
    for (int i = 0; i < G::NBAR; ++i) {
      uint32_t cnt = 1;
      if (i >= G::B_XFORM && i < G::B_XFORM + NS) cnt = 64;
      else if ((i >= G::B_QREADY && i < G::B_QREADY + NS) || (i >= G::B_PFULL && i < G::B_PFULL + 2) ||
               (i >= G::B_OEMPTY && i < G::B_OEMPTY + 2) || i == G::B_UREADY || i == G::B_SBFULL)
        cnt = 128;
      mbar_init(bars + i, cnt);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_u);
  }
  if (warp == 1) tmem_alloc(tmem_slot, G::T_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp < 4) {
    reg_dealloc<104>();
    if (warp == 0 && lane == 0) {
      // ============================================================ TMA producer
      int issued = 0;
      for (int c = 0; c < nchunks; ++c) {
        const int s = c % NS, k = c / NS;
        if (!wait_bar(sy, G::B_EMPTY + s, (k & 1) ^ 1, c)) break;
        mbar_arrive_expect_tx(bars + G::B_FULL + s, G::LOAD_BYTES);
        const int t0 = (int)(sq.start + (int64_t)c * kC);
        const int bi = (int)sq.bidx;
        uint8_t *st = stage(s);
        const int64_t slot = (a.coff ? (int64_t)a.coff[n] : n * a.nck) + c;
        bulk_load(dtab + s * G::DT_STRIDE, a.bt + (slot * a.H + h) * G::DT_STRIDE, G::DT_STRIDE * 4,
                  bars + G::B_FULL + s);
        for (int kb = 0; kb < 2; ++kb) {
          tma_load_4d(st + G::OFF_Q + kb * kSlab, &tm_q, bars + G::B_FULL + s, kb * 64, h, t0, bi);
          tma_load_4d(st + G::OFF_K + kb * kSlab, &tm_k, bars + G::B_FULL + s, kb * 64, h, t0, bi);
          tma_load_4d(st + G::OFF_W + kb * kSlab, &tm_w, bars + G::B_FULL + s, kb * 64, h, t0, bi);
          tma_load_4d(st + G::OFF_U + kb * kSlab, &tm_u, bars + G::B_FULL + s, kb * 64, h, t0, bi);
        }
        issued = c + 1;
      }
      if (*abort_flag) {  // let every issued copy land before the CTA exits
        for (int c = max(0, issued - NS); c < issued; ++c) drain_bar(sy, G::B_FULL + c % NS, (c / NS) & 1);
      }
    } else if (warp == 1 && lane == 0) {
      // ============================================================ MMA issuer
      constexpr uint32_t ID_S = idesc_bf16_f32(kC, kC, 0, 0);   // scores
      constexpr uint32_t ID_O = idesc_bf16_f32(kC, kD, 0, 1);   // WS, O
      constexpr uint32_t ID_U = idesc_bf16_f32(kD, kD, 1, 1);   // state update
      const uint64_t dsb = smem_desc_sw128(smem_u32(sm + G::OFF_SB), G::SB_SLAB, 1024);
      // operand descriptors of stage 0; stage s adds s * STAGE_BYTES / 16 to the
      // start-address field (no carry: shared addresses are < 256 KB)
      const uint64_t dq0 = smem_desc_sw128(smem_u32(stage(0) + G::OFF_Q), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_u32(stage(0) + G::OFF_K), 16, 1024);
      const uint64_t dw0 = smem_desc_sw128(smem_u32(stage(0) + G::OFF_W), 16, 1024);
      const uint64_t du0 = smem_desc_sw128(smem_u32(stage(0) + G::OFF_U), kSlab, 1024);   // MN-major
      const uint64_t dkd0 = smem_desc_sw128(smem_u32(stage(0) + G::OFF_KD), kSlab, 1024); // MN-major
      const uint64_t dp0 = smem_desc_sw128(smem_u32(sm + G::OFF_P), 16, 1024);
      auto soff = [](int s) -> uint64_t { return (uint64_t)(s * (G::STAGE_BYTES >> 4)); };
      int m1_issued = 0;
      // The last commit: its arrival means every product issued before it has finished.
      int last_bar = -1;
      uint32_t last_par = 0;
      auto commit = [&](int idx, uint32_t parity) {
        umma_commit(bars + idx);
        last_bar = idx;
        last_par = parity;
      };
      // M1 of chunk c: A[c & 1] = Q K^T (raw keys)
      auto issue_scores = [&](int c) -> bool {
        const int s = c % NS, k = c / NS, b = c & 1;
        if (!wait_bar(sy, G::B_FULL + s, k & 1, c)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          umma_bf16(tbase + G::T_A + b * kC, dq0 + soff(s) + kmaj(kk), dk0 + soff(s) + kmaj(kk), ID_S, kk > 0);
        commit(G::B_AFULL + b, (c >> 1) & 1);
        m1_issued = c + 1;
        return true;
      };
      constexpr bool kEarlyM2 = false;
      // M2 of chunk c: O = Qd Sb
      auto issue_m2 = [&](int c) {
        const int s = c % NS, b = c & 1;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          umma_bf16(tbase + G::T_O + b * kD, dq0 + soff(s) + kmaj(kk), dsb + ((kk * 2048) >> 4), ID_O, kk > 0);
        commit(G::B_SBEMPTY, sbi(c) & 1);
      };
      // Per chunk: MW; then, while the state warps compute U, the next chunk's M1 as
      // soon as its tiles have landed (the tensor pipe is idle there; issued later it
      // would queue in front of the next MW); M4 at UREADY; M2, M3; the next M1 now if
      // its tiles were late.
      const bool started = nchunks == 0 || issue_scores(0);
      for (int c = 0; c < nchunks && started; ++c) {
        const int s = c % NS, k = c / NS, b = c & 1;
        const uint32_t o_acc = tbase + G::T_O + b * kD;
        bool ok = true, m2 = false;
        // MW: WS = W Sb
        if (prev(c)) {
          ok = wait_bar(sy, G::B_FULL + s, k & 1, c) && wait_bar(sy, G::B_SBFULL, sbi(c) & 1, c);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk)
            umma_bf16(tbase + G::T_U, dw0 + soff(s) + kmaj(kk), dsb + ((kk * 2048) >> 4), ID_O, kk > 0);
          commit(G::B_WSFULL, sbi(c) & 1);
        }
        {
          const int c1 = c + 1, s1 = c1 % NS, k1 = c1 / NS;
          bool m1n = c1 >= nchunks;
          const long long t0 = clock64();
          while (!mbar_test(bars + G::B_UREADY, c & 1) && !*abort_flag && clock64() - t0 < kTimeoutCycles) {
            if (!m1n && mbar_test(bars + G::B_FULL + s1, k1 & 1)) m1n = issue_scores(c1);
            if (kEarlyM2 && prev(c) && !m2 && mbar_test(bars + G::B_OEMPTY + b, ((c >> 1) & 1) ^ 1) &&
                mbar_test(bars + G::B_QREADY + s, k & 1)) {
              issue_m2(c);
              m2 = true;
            }
          }
        }
        // M4: Us = Kd^T U
        if (!wait_bar(sy, G::B_UREADY, c & 1, c)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk)
          umma_bf16(tbase + G::T_U, dkd0 + soff(s) + ((kk * 2048) >> 4), du0 + soff(s) + ((kk * 2048) >> 4), ID_U,
                    kk > 0);
        commit(G::B_UFULL, c & 1);
        // M2: O = Qd Sb.  Qd is waited for even without M2: the output warps write
        // it in place, so the stage must not be released before they are done.
        if (!wait_bar(sy, G::B_OEMPTY + b, ((c >> 1) & 1) ^ 1, c) || !wait_bar(sy, G::B_QREADY + s, k & 1, c))
          break;
        if (prev(c) && !m2) issue_m2(c);
        // M3: O += P U
        if (!wait_bar(sy, G::B_PFULL + b, (c >> 1) & 1, c)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk)
          umma_bf16(o_acc, dp0 + (uint64_t)(b * (kSlab >> 4)) + kmaj(kk), du0 + soff(s) + ((kk * 2048) >> 4),
                    ID_O, (prev(c) || kk > 0) ? 1u : 0u);
        commit(G::B_OFULL + b, (c >> 1) & 1);
        commit(G::B_EMPTY + s, k & 1);
        if (m1_issued < c + 2 && c + 1 < nchunks && !issue_scores(c + 1)) break;
      }
      // the last commits arrive asynchronously: wait for them before tensor memory is freed
      if (last_bar >= 0) drain_bar(sy, last_bar, last_par);
    } else if (warp >= 2) {
      // ========================================================== transform
      // 64 threads; thread tt owns the 16-byte vectors tt + 64 m (m < 8) of both
      // 64-column slabs of the key tile: row tt/8 + 8 m, physical chunk tt mod 8.
      // Kd = diag(e^{b_last - b} / |k|) K (= diag(e^{b_last - b}) Kt), zero past the chunk end.
      const int tt = tid - 64;
      for (int c = 0; c < nchunks; ++c) {
        const int s = c % NS, k = c / NS;
        if (!wait_bar_warp(sy, G::B_FULL + s, k & 1, c)) break;
        const int Cp = chunk_len(c);
        const float *dt = dtab + s * G::DT_STRIDE;
        const float blast = dt[kC - 1];
        const uint8_t *kt = stage(s) + G::OFF_K;
        uint8_t *kd = stage(s) + G::OFF_KD;
#pragma unroll 2
        for (int m = 0; m < 8; ++m) {
          const int r = (tt >> 3) + 8 * m;
          const int off = (tt + 64 * m) * 16;
          const float wd = r < Cp ? exp_fast(blast + dt[kC + r]) : 0.f;
#pragma unroll
          for (int sl = 0; sl < 2; ++sl) {
            float f[8];
            unpack8(*reinterpret_cast<const uint4 *>(kt + sl * kSlab + off), f);
#pragma unroll
            for (int u = 0; u < 8; ++u) f[u] = r < Cp ? f[u] * wd : 0.f;
            *reinterpret_cast<uint4 *>(kd + sl * kSlab + off) = pack8(f);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(bars + G::B_XFORM + s);
      }
    }
  } else if (warp < 8) {
    // ================================================================ state
    reg_alloc<232>();
    const int sp = warp & 3;
    const int kr = sp * 32 + lane;  // row of S^T (d_k index) held by this thread
    const uint32_t lane_base = tbase + ((uint32_t)(sp * 32) << 16);
    const int64_t sbase = (n * a.H + h) * (int64_t)a.dk * a.dv;
    float S[kD];
    if (has_init) {
      const float4 *src = reinterpret_cast<const float4 *>(a.init + sbase + (int64_t)kr * a.dv);
#pragma unroll
      for (int q = 0; q < kD / 4; ++q) {
        const float4 x = (kr < a.dk && 4 * q < a.dv) ? src[q] : make_float4(0.f, 0.f, 0.f, 0.f);
        S[4 * q] = x.x;
        S[4 * q + 1] = x.y;
        S[4 * q + 2] = x.z;
        S[4 * q + 3] = x.w;
      }
    } else {
#pragma unroll
      for (int u = 0; u < kD; ++u) S[u] = 0.f;
    }
    // Sb = bf16(S^T): two [d_k x 64] slabs, MN-major (row kr, 128-byte swizzle)
    auto write_sb = [&]() {
#pragma unroll
      for (int grp = 0; grp < kD / 32; ++grp) {
        uint8_t *row = sm + G::OFF_SB + (grp >> 1) * G::SB_SLAB + kr * 128;
        const int ch0 = (grp & 1) * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float *x = &S[grp * 32 + 8 * q];
          *reinterpret_cast<uint4 *>(row + (((ch0 + q) ^ (kr & 7)) << 4)) =
              make_uint4(pack2(x[0], x[1]), pack2(x[2], x[3]), pack2(x[4], x[5]), pack2(x[6], x[7]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bars + G::B_SBFULL);
    };
    const int i = sp * 16 + (lane & 15), hf = lane >> 4;  // U row and column half of this thread
    float gdec = 1.f;  // e^{b_last} of the previous chunk
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const int s = c % NS, k = c / NS;
      ok = false;
      if (c > 0) {  // S^T <- e^{b_last} S^T + Us of chunk c - 1 (two loads in flight per wait)
        if (!wait_bar_warp(sy, G::B_UFULL, (c - 1) & 1, c)) break;
        tc_fence_after();
#pragma unroll
        for (int grp = 0; grp < kD / 32; grp += 2) {
          uint32_t r0[32], r1[32];
          tmem_ld_32x32b_x32(lane_base + G::T_U + grp * 32, r0);
          tmem_ld_32x32b_x32(lane_base + G::T_U + grp * 32 + 32, r1);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            S[grp * 32 + e] = fmaf(gdec, S[grp * 32 + e], __uint_as_float(r0[e]));
            S[grp * 32 + 32 + e] = fmaf(gdec, S[grp * 32 + 32 + e], __uint_as_float(r1[e]));
          }
        }
      }
      if (prev(c)) {  // Sb of chunk c, once the products of chunk c - 1 have read the previous one
        if (sbi(c) >= 1 && !wait_bar_warp(sy, G::B_SBEMPTY, (sbi(c) - 1) & 1, c)) break;
        write_sb();
      }
      if (!wait_bar_warp(sy, G::B_FULL + s, k & 1, c) || !wait_bar_warp(sy, G::B_XFORM + s, k & 1, c)) break;
      const float blast = dtab[s * G::DT_STRIDE + kC - 1];
      const int Cp = chunk_len(c);
      // U = Ut - WS on row i, columns [64 hf, 64 hf + 64), in place; zero past the chunk end.
      // The Ut row is read while the product still runs.
      uint8_t *urow = stage(s) + G::OFF_U + hf * kSlab;
      uint4 ut[8];
#pragma unroll
      for (int p = 0; p < 8; ++p) ut[p] = *reinterpret_cast<const uint4 *>(urow + swz(i, p));
      if (prev(c)) {
        if (!wait_bar_warp(sy, G::B_WSFULL, sbi(c) & 1, c)) break;
        tc_fence_after();
      }
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        uint32_t r[32];
        if (prev(c)) {
          tmem_ld_16x32bx2_x32<64>(lane_base + G::T_U + pass * 32, r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = 0u;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float f[8];
          unpack8(ut[pass * 4 + q], f);
#pragma unroll
          for (int u = 0; u < 8; ++u) f[u] = i < Cp ? f[u] - __uint_as_float(r[8 * q + u]) : 0.f;
          *reinterpret_cast<uint4 *>(urow + swz(i, pass * 4 + q)) = pack8(f);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bars + G::B_UREADY);
      gdec = exp_fast(blast);
      ok = true;
    }
    // the last chunk's update, then the final state (zero for an empty sequence)
    if (ok && nchunks > 0 && wait_bar_warp(sy, G::B_UFULL, (nchunks - 1) & 1, nchunks)) {
      tc_fence_after();
#pragma unroll
      for (int grp = 0; grp < kD / 32; ++grp) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(lane_base + G::T_U + grp * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) S[grp * 32 + e] = fmaf(gdec, S[grp * 32 + e], __uint_as_float(r[e]));
      }
    }
    if (a.final_state && !*abort_flag && kr < a.dk) {
      float4 *dst = reinterpret_cast<float4 *>(a.final_state + sbase + (int64_t)kr * a.dv);
#pragma unroll
      for (int q = 0; q < kD / 4; ++q)
        if (4 * q < a.dv) dst[q] = make_float4(S[4 * q], S[4 * q + 1], S[4 * q + 2], S[4 * q + 3]);
    }
  } else {
    // ================================================================ output
    const int sp = warp & 3;
    const int i = sp * 16 + (lane & 15), hf = lane >> 4;  // chunk row and column half of this thread
    const uint32_t lane_base = tbase + ((uint32_t)(sp * 32) << 16);
    uint8_t *obase = reinterpret_cast<uint8_t *>(a.out) + 2 * (sq.bidx * a.o_sb + (int64_t)h * a.o_sh);

    // chunk c: P = tril(A) .* D into P[c & 1], then Qd = diag(e^b) Q in place
    auto scores = [&](int c) -> bool {
      const int s = c % NS, k = c / NS, b = c & 1;
      const int Cp = chunk_len(c);
      if (!wait_bar_warp(sy, G::B_AFULL + b, (c >> 1) & 1, c)) return false;
      tc_fence_after();
      if (!wait_bar_warp(sy, G::B_FULL + s, k & 1, c)) return false;
      const float *dt = dtab + s * G::DT_STRIDE;
      const float bi = dt[i];
      uint32_t r[32];
      tmem_ld_16x32bx2_x32<32>(lane_base + G::T_A + b * kC, r);
      tmem_wait_ld();
      float f[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int j = hf * 32 + e;
        f[e] = (j <= i && i < Cp) ? __uint_as_float(r[e]) * exp_fast(bi + dt[kC + j]) : 0.f;
      }
      uint8_t *prow = sm + G::OFF_P + b * kSlab;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4 *>(prow + swz(i, hf * 4 + q)) =
            make_uint4(pack2(f[8 * q], f[8 * q + 1]), pack2(f[8 * q + 2], f[8 * q + 3]),
                       pack2(f[8 * q + 4], f[8 * q + 5]), pack2(f[8 * q + 6], f[8 * q + 7]));
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bars + G::B_PFULL + b);  // also tells the MMA issuer that A[b] has been read
      // the score product has read Q: scale its row i by e^{b_i} for the inter-chunk product
      // (chunks in swizzled order, so that the rows of a warp spread over the banks)
      const float qf = i < Cp ? exp_fast(bi) : 0.f;
      uint8_t *qrow = stage(s) + G::OFF_Q + hf * kSlab;
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        uint4 *p4 = reinterpret_cast<uint4 *>(qrow + swz(i, p));
        float x[8];
        unpack8(*p4, x);
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] *= qf;
        *p4 = pack8(x);
      }
      fence_proxy_async_smem();
      mbar_arrive(bars + G::B_QREADY + s);
      return true;
    };

    // epilogue of chunk c: O[c & 1] -> bf16 output rows
    auto epilogue = [&](int c) -> bool {
      const int b = c & 1;
      const int Cp = chunk_len(c);
      if (!wait_bar_warp(sy, G::B_OFULL + b, (c >> 1) & 1, c)) return false;
      tc_fence_after();
      const int64_t tok = sq.start + (int64_t)c * kC + i;
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        uint32_t r[32];
        tmem_ld_16x32bx2_x32<64>(lane_base + G::T_O + b * kD + pass * 32, r);
        tmem_wait_ld();
        if (pass == 1) {
          tc_fence_before();
          mbar_arrive(bars + G::B_OEMPTY + b);
        }
        if (i < Cp && hf * 64 + pass * 32 < a.dv) {
          uint4 *dst = reinterpret_cast<uint4 *>(obase + 2 * (tok * a.o_st + hf * 64 + pass * 32));
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack2(__uint_as_float(r[8 * q]), __uint_as_float(r[8 * q + 1])),
                                pack2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3])),
                                pack2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5])),
                                pack2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7])));
        }
      }
      return true;
    };

    for (int t = 0; t <= nchunks; ++t) {
      if (t < nchunks && !scores(t)) break;
      if (t >= 1 && !epilogue(t - 1)) break;
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    tmem_dealloc(tbase, G::T_COLS);
    tmem_relinquish();
  }
}

}  // namespace

// ---------------------------------------------------------------- host side
namespace {

constexpr int kStages = 2;

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace regions, in order: W and Ut (bf16 [B, T, H, 128] each), the chunk
// tables ([chunk slot][H][2][C] fp32: b_i, ln(1/|k_i|) - b_i) and, for packed batches, the
// first chunk slot of each sequence.  Packed batches bound their slot count by
// ceil(T / C) + n_seqs (each sequence adds at most one partial chunk).
struct WsPlan {
  size_t wu, bt, coff, total;
  int64_t nck, slots;
};
WsPlan ws_plan(int64_t B, int64_t T, int64_t H, int64_t n_seqs, bool varlen) {
  WsPlan p;
  p.nck = (T + kC - 1) / kC;
  p.slots = varlen ? p.nck + n_seqs : n_seqs * p.nck;
  p.wu = align256((size_t)(B * T * H) * kD * 2);
  p.bt = align256((size_t)(p.slots * H) * 2 * kC * 4);
  p.coff = varlen ? align256((size_t)(n_seqs + 1) * 4) : 0;
  p.total = 2 * p.wu + p.bt + p.coff;
  return p;
}

}  // namespace

// Head dims of the tensor-core path: 64 or 128 each (a 64 in the 128 layout, zero padded).
bool gdn_shape(int dk, int dv) { return (dk == 64 || dk == kD) && (dv == 64 || dv == kD); }

bool gdn_tc_supported(const DeltaArgs &a) { return a.dtype == LA_BF16 && gdn_shape(a.dk, a.dv); }

size_t gdn_workspace_bytes(int64_t B, int64_t T, int64_t H, int dk, int dv, int64_t n_seqs, bool varlen) {
  if (!gdn_shape(dk, dv)) return 0;
  return ws_plan(B, T, H, n_seqs, varlen).total;
}

cudaError_t launch_gdn_chunk(const DeltaArgs &a, void *workspace, size_t workspace_bytes, cudaStream_t stream,
                             const char **why) {
  const int64_t B = a.cu_seqlens ? 1 : a.n_seqs;
  const bool varlen = a.cu_seqlens != nullptr;
  const WsPlan plan = ws_plan(B, a.T, a.H, a.n_seqs, varlen);
  if (!workspace || workspace_bytes < plan.total) {
    if (why) *why = "workspace too small for the chunked gated delta rule";
    return cudaErrorInvalidValue;
  }
  if (plan.slots * a.H > 0x7fffffffLL || a.n_seqs * a.H > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  __nv_bfloat16 *w = reinterpret_cast<__nv_bfloat16 *>(ws);
  __nv_bfloat16 *ut = reinterpret_cast<__nv_bfloat16 *>(ws + plan.wu);
  float *bt = reinterpret_cast<float *>(ws + 2 * plan.wu);
  int32_t *coff = varlen ? reinterpret_cast<int32_t *>(ws + 2 * plan.wu + plan.bt) : nullptr;
  const TensorView wv{w, a.T * a.H * kD, (int64_t)a.H * kD, kD};
  const TensorView uv{ut, a.T * a.H * kD, (int64_t)a.H * kD, kD};
  CUtensorMap mq, mk, mv, mw, mu;
  // q, k, v maps have the tensors' own head dims: columns past them read as zero fill
  if (!make_map(&mq, a.q, B, a.T, a.H, a.dk, kC) || !make_map(&mk, a.k, B, a.T, a.H, a.dk, kC) ||
      !make_map(&mv, a.v, B, a.T, a.H, a.dv, kC) || !make_map(&mw, wv, B, a.T, a.H, kD, kC) ||
      !make_map(&mu, uv, B, a.T, a.H, kD, kC)) {
    if (why) *why = "cuTensorMapEncodeTiled rejected a tensor";
    return cudaErrorInvalidValue;
  }
  cudaError_t err;
  // 1. the per-chunk WY pass (grid: chunk slots x heads)
  if (plan.slots > 0 && a.T > 0) {
    if (varlen) {
      gdn_chunk_offsets_kernel<<<1, 1024, 0, stream>>>(a.cu_seqlens, a.n_seqs, coff);
      if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    PrepArgs p;
    p.g = a.g;
    p.beta = a.beta;
    p.cu_seqlens = a.cu_seqlens;
    p.coff = coff;
    p.w = w;
    p.ut = ut;
    p.bt = bt;
    p.T = a.T;
    p.n_seqs = a.n_seqs;
    p.H = a.H;
    p.skip_load = a.test_wait_timeout ? 1 : 0;
    err = cudaFuncSetAttribute(gdn_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PrepCfg::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    gdn_prep_kernel<<<(unsigned)(plan.slots * a.H), 128, PrepCfg::SMEM_BYTES, stream>>>(mk, mv, p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  // 2. the sequential pass, one CTA per (sequence, head)
  GdnTcArgs t;
  t.out = a.out;
  t.o_sb = a.o_sb;
  t.o_st = a.o_st;
  t.o_sh = a.o_sh;
  t.bt = bt;
  t.coff = coff;
  t.nck = plan.nck;
  t.init = a.init;
  t.final_state = a.final_state;
  t.cu_seqlens = a.cu_seqlens;
  t.T = a.T;
  t.H = a.H;
  t.dk = a.dk;
  t.dv = a.dv;
  using G = GdnCfg<kStages>;
  auto kern = gdn_tc_kernel<kStages>;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM_BYTES);
  if (err != cudaSuccess) return err;
  kern<<<(unsigned)(a.n_seqs * a.H), kThreads, G::SMEM_BYTES, stream>>>(mq, mk, mw, mu, t);
  return cudaGetLastError();
}

cudaError_t gdn_device_error(unsigned int *flags, unsigned int *where, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(flags, g_gdn_error, sizeof(unsigned int));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(where, g_gdn_where, sizeof(unsigned int));
  if (e == cudaSuccess && reset) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_gdn_error, &zero, sizeof(zero));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_gdn_where, &zero, sizeof(zero));
  }
  return e;
}

}  // namespace la
