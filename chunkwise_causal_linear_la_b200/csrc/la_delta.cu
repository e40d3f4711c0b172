// la_delta.cu -- the gated delta rule, token by token on CUDA cores (fp32).
//
// "1.6 长上下文与高效注意力", section Gated delta rule: with the key normalised
// to unit length (kt = k_t / max(|k_t|, 1e-12), as in the section's listing),
//     S_t = alpha_t S_{t-1} (I - beta_t kt kt^T) + beta_t v_t kt^T,   o_t = S_t q_t,
// alpha_t = exp(g_t).  Row r of S (the state of value column r) evolves on its
// own: with u_r = S[r, :] . kt,
//     S[r, :] <- alpha S[r, :] + beta (v_r - alpha u_r) kt,    o_r = S[r, :] . q_t,
// so the P adjacent lanes of a column each hold d_k / P of its state values in
// registers, interleaved by 16-byte granules (lane p of a column holds the
// granules p, p + P, ..., so the warp's broadcast loads of the key and query
// hit distinct banks), and the dot products finish with log2 P shuffles and the columns of
// a head are split over CTAs freely: 128 columns per CTA of 128 P threads.
// Splitting d_k shortens each thread's per-token chain, which is what bounds
// this token-by-token kernel.  Each CTA stages a tile of C tokens of q, the unit keys,
// v, alpha and beta in shared memory (read by every thread as broadcasts) and
// then walks the tile's tokens in order.
#include <cuda_bf16.h>

#include "la_common.cuh"
#include "la_internal.h"

namespace la {
namespace {

constexpr int kDeltaCols = 128;  // value columns per CTA
constexpr int kDeltaTile = 64;

// KP: state values per thread; P: threads per value column (KP * P = d_k)
template <typename Tin, int KP, int P>
__global__ void __launch_bounds__(kDeltaCols * P)
delta_kernel(DeltaArgs a) {
  extern __shared__ float sm[];
  constexpr int kDeltaThreads = kDeltaCols * P;
  constexpr int DK = KP * P;
  constexpr int COLS = kDeltaCols;
  float *qs = sm;                          // [C][DK]
  float *ks = qs + kDeltaTile * DK;        // [C][DK] unit keys
  float *vs = ks + kDeltaTile * DK;        // [C][COLS]
  float *al = vs + kDeltaTile * COLS;      // [C] alpha
  float *be = al + kDeltaTile;             // [C] beta

  const int tid = threadIdx.x;
  const int nsl = (a.dv + COLS - 1) / COLS;
  const int64_t unit = blockIdx.x;
  const int sl = (int)(unit % nsl);
  const int h = (int)((unit / nsl) % a.H);
  const int64_t n = unit / ((int64_t)nsl * a.H);
  const int p = tid % P, col = tid / P;
  const int r = sl * COLS + col;  // value column of this thread
  const bool active = r < a.dv;
  int64_t b, start, len;
  if (a.cu_seqlens) {
    b = 0;
    start = a.cu_seqlens[n];
    len = (int64_t)a.cu_seqlens[n + 1] - start;
  } else {
    b = n;
    start = 0;
    len = a.T;
  }
  const Tin *Q = (const Tin *)a.q.data + b * a.q.sb + h * a.q.sh;
  const Tin *K = (const Tin *)a.k.data + b * a.k.sb + h * a.k.sh;
  const Tin *V = (const Tin *)a.v.data + b * a.v.sb + h * a.v.sh;
  Tin *O = (Tin *)a.out + b * a.o_sb + h * a.o_sh;
  const int64_t srow = b * a.T + start;  // first token row of the sequence in [B * T]

  float S[KP];  // S[4 j + e] is state row 4 (p + P j) + e of column r
  const int64_t sbase = ((int64_t)n * a.H + h) * (int64_t)DK * a.dv;
  auto krow = [&](int c) -> int { return 4 * (p + P * (c >> 2)) + (c & 3); };
#pragma unroll
  for (int c = 0; c < KP; ++c) S[c] = (a.init && active) ? a.init[sbase + (int64_t)krow(c) * a.dv + r] : 0.f;

  for (int64_t t0 = 0; t0 < len; t0 += kDeltaTile) {
    const int Ct = (int)min((int64_t)kDeltaTile, len - t0);
    __syncthreads();  // the previous tile is consumed
    for (int e = tid; e < Ct * DK; e += kDeltaThreads) {
      const int i = e / DK, c = e % DK;
      const int64_t t = start + t0 + i;
      qs[e] = to_f32<Tin>(Q[t * a.q.st + c]);
      ks[e] = to_f32<Tin>(K[t * a.k.st + c]);
    }
    for (int e = tid; e < Ct * COLS; e += kDeltaThreads) {
      const int i = e / COLS, cc = e % COLS, rr = sl * COLS + cc;
      vs[e] = rr < a.dv ? to_f32<Tin>(V[(start + t0 + i) * a.v.st + rr]) : 0.f;
    }
    for (int i = tid; i < Ct; i += kDeltaThreads) {
      const int64_t row = (srow + t0 + i) * a.H + h;
      al[i] = expf(a.g[row]);
      be[i] = a.beta[row];
    }
    __syncthreads();
    // unit keys: one warp per row
    for (int i = tid >> 5; i < Ct; i += kDeltaThreads / 32) {
      float ss = 0.f;
      for (int c = tid & 31; c < DK; c += 32) ss = fmaf(ks[i * DK + c], ks[i * DK + c], ss);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv = 1.f / fmaxf(sqrtf(ss), 1e-12f);
      for (int c = tid & 31; c < DK; c += 32) ks[i * DK + c] *= inv;
    }
    __syncthreads();
    for (int i = 0; i < Ct; ++i) {
      const float *kt = ks + i * DK;
      const float *qt = qs + i * DK;
      static_assert(KP % 4 == 0, "16-byte broadcast loads of the key and query");
      const float4 *kt4 = reinterpret_cast<const float4 *>(kt);
      const float4 *qt4 = reinterpret_cast<const float4 *>(qt);
      float u0 = 0.f, u1 = 0.f, u2 = 0.f, u3 = 0.f;
#pragma unroll
      for (int c = 0; c < KP; c += 4) {
        const float4 kv = kt4[p + P * (c / 4)];
        u0 = fmaf(S[c], kv.x, u0);
        u1 = fmaf(S[c + 1], kv.y, u1);
        u2 = fmaf(S[c + 2], kv.z, u2);
        u3 = fmaf(S[c + 3], kv.w, u3);
      }
      float u = (u0 + u1) + (u2 + u3);
#pragma unroll
      for (int m = 1; m < P; m <<= 1) u += __shfl_xor_sync(0xffffffffu, u, m);
      __syncwarp();  // reload kt below instead of keeping all of it in registers
      const float alpha = al[i];
      const float coef = be[i] * (vs[i * COLS + col] - alpha * u);
      float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
#pragma unroll
      for (int c = 0; c < KP; c += 4) {
        const float4 kv = kt4[p + P * (c / 4)];
        const float4 qv = qt4[p + P * (c / 4)];
        S[c] = fmaf(alpha, S[c], coef * kv.x);
        S[c + 1] = fmaf(alpha, S[c + 1], coef * kv.y);
        S[c + 2] = fmaf(alpha, S[c + 2], coef * kv.z);
        S[c + 3] = fmaf(alpha, S[c + 3], coef * kv.w);
        o0 = fmaf(S[c], qv.x, o0);
        o1 = fmaf(S[c + 1], qv.y, o1);
        o2 = fmaf(S[c + 2], qv.z, o2);
        o3 = fmaf(S[c + 3], qv.w, o3);
      }
      float o = (o0 + o1) + (o2 + o3);
#pragma unroll
      for (int m = 1; m < P; m <<= 1) o += __shfl_xor_sync(0xffffffffu, o, m);
      if (p == 0 && active) O[(start + t0 + i) * a.o_st + r] = from_f32<Tin>(o);
    }
  }
  if (a.final_state && active) {
#pragma unroll
    for (int c = 0; c < KP; ++c) a.final_state[sbase + (int64_t)krow(c) * a.dv + r] = S[c];
  }
}

template <typename Tin, int KP, int P>
cudaError_t launch_kp(const DeltaArgs &a, cudaStream_t stream) {
  constexpr int COLS = kDeltaCols;
  constexpr int kDeltaThreads = kDeltaCols * P;
  const int64_t grid = a.n_seqs * a.H * ((a.dv + COLS - 1) / COLS);
  if (grid == 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const size_t smem = (size_t)(2 * kDeltaTile * KP * P + kDeltaTile * COLS + 2 * kDeltaTile) * sizeof(float);
  auto kern = delta_kernel<Tin, KP, P>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  kern<<<(unsigned)grid, kDeltaThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_dtype(const DeltaArgs &a, cudaStream_t stream) {
  switch (a.dk) {
    case 16: return launch_kp<Tin, 16, 1>(a, stream);
    case 32: return launch_kp<Tin, 16, 2>(a, stream);
    case 64: return launch_kp<Tin, 16, 4>(a, stream);
    case 128: return launch_kp<Tin, 32, 4>(a, stream);
    case 256: return launch_kp<Tin, 64, 4>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

// One token per sequence (decode): the state is read once and written once, so the
// kernel is built for coalesced state traffic instead.  One CTA of 128 threads per
// (sequence, head, 32 value columns): thread (row group rg, column quad cq) holds
// rows rg, rg + 16, ... of S^T for columns 4 cq .. 4 cq + 3, all requested with
// streaming loads before anything else (a warp moves 4 rows x 128 contiguous bytes
// per instruction).  Both reductions over d_k come out of one pass over the old
// state: with coef_r = beta (v_r - alpha u_r), the output of the updated state is
// o = S_new q = alpha (S^T-contract q) + coef (kt . q), so u = S^T-contract kt and
// p = S^T-contract q are summed over the 16 row groups together, behind a single
// barrier.  Small CTAs keep the whole grid resident: the 512-thread CTAs used
// before ran the [256, 4, 128, 128] state in 3.5 waves.
constexpr int kDecThreads = 128;
constexpr int kDecCols = 32;                       // value columns per CTA
constexpr int kDecQuads = kDecCols / 4;            // float4 column quads
constexpr int kDecGroups = kDecThreads / kDecQuads;  // row groups (16)
template <typename Tin, int DK>
__global__ void __launch_bounds__(kDecThreads) delta_decode_kernel(DeltaArgs a) {
  constexpr int RW = DK / kDecGroups;  // rows of S^T per thread
  __shared__ float kt[DK], qv[DK];
  __shared__ float4 pu[kDecGroups][kDecQuads], pq[kDecGroups][kDecQuads];
  __shared__ float red[2][kDecThreads / 32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cq = tid % kDecQuads, rg = tid / kDecQuads;
  const int nsl = (a.dv + kDecCols - 1) / kDecCols;
  const int64_t unit = blockIdx.x;
  const int sl = (int)(unit % nsl);
  const int h = (int)((unit / nsl) % a.H);
  const int64_t n = unit / ((int64_t)nsl * a.H);
  const int64_t b = n, t = 0;  // the sequence's one token
  const int r0 = sl * kDecCols + 4 * cq;
  const bool active = r0 < a.dv;  // dv is a multiple of 4
  const int64_t sbase = ((int64_t)n * a.H + h) * (int64_t)DK * a.dv;
  float4 S[RW];
#pragma unroll
  for (int j = 0; j < RW; ++j)
    S[j] = (a.init && active)
               ? __ldcs(reinterpret_cast<const float4 *>(a.init + sbase + (int64_t)(rg + kDecGroups * j) * a.dv + r0))
               : make_float4(0.f, 0.f, 0.f, 0.f);
  const Tin *Q = (const Tin *)a.q.data + b * a.q.sb + t * a.q.st + h * a.q.sh;
  const Tin *K = (const Tin *)a.k.data + b * a.k.sb + t * a.k.st + h * a.k.sh;
  const Tin *V = (const Tin *)a.v.data + b * a.v.sb + t * a.v.st + h * a.v.sh;
  const int64_t row = (b * a.T + t) * a.H + h;
  const float alpha = expf(a.g[row]), beta = a.beta[row];
  // raw key and query in shared memory, |k|^2 and k . q
  float ss = 0.f, kq = 0.f;
  for (int c = tid; c < DK; c += kDecThreads) {
    const float kv = to_f32<Tin>(K[c]), qq = to_f32<Tin>(Q[c]);
    kt[c] = kv;
    qv[c] = qq;
    ss = fmaf(kv, kv, ss);
    kq = fmaf(kv, qq, kq);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    kq += __shfl_xor_sync(0xffffffffu, kq, o);
  }
  if (lane == 0) {
    red[0][warp] = ss;
    red[1][warp] = kq;
  }
  float4 vv = make_float4(0.f, 0.f, 0.f, 0.f);
  if (active) vv = make_float4(to_f32<Tin>(V[r0]), to_f32<Tin>(V[r0 + 1]), to_f32<Tin>(V[r0 + 2]), to_f32<Tin>(V[r0 + 3]));
  __syncthreads();
  // this thread's rows of u = sum_c k_c S^T[c][:] (raw key) and p = sum_c q_c S^T[c][:]
  float4 u = make_float4(0.f, 0.f, 0.f, 0.f), p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j = 0; j < RW; ++j) {
    const int c = rg + kDecGroups * j;
    const float kc = kt[c], qc = qv[c];
    u.x = fmaf(kc, S[j].x, u.x);
    u.y = fmaf(kc, S[j].y, u.y);
    u.z = fmaf(kc, S[j].z, u.z);
    u.w = fmaf(kc, S[j].w, u.w);
    p.x = fmaf(qc, S[j].x, p.x);
    p.y = fmaf(qc, S[j].y, p.y);
    p.z = fmaf(qc, S[j].z, p.z);
    p.w = fmaf(qc, S[j].w, p.w);
  }
  pu[rg][cq] = u;
  pq[rg][cq] = p;
  __syncthreads();
  float sst = 0.f, kqt = 0.f;
#pragma unroll
  for (int w = 0; w < kDecThreads / 32; ++w) {
    sst += red[0][w];
    kqt += red[1][w];
  }
  const float inv = 1.f / fmaxf(sqrtf(sst), 1e-12f);  // kt = k inv, the listing's floor on |k|
  u = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int r = 0; r < kDecGroups; ++r) {
    const float4 x = pu[r][cq];
    u.x += x.x;
    u.y += x.y;
    u.z += x.z;
    u.w += x.w;
  }
  // S <- alpha (S - beta kt u^T) + beta kt v^T, i.e. S^T[c][r] = alpha S^T[c][r] + coef_r kt_c
  // with u taken with the unit key and coef_r = beta (v_r - alpha u_r)
  const float4 coef = make_float4(beta * (vv.x - alpha * u.x * inv), beta * (vv.y - alpha * u.y * inv),
                                  beta * (vv.z - alpha * u.z * inv), beta * (vv.w - alpha * u.w * inv));
  if (a.final_state && active) {
#pragma unroll
    for (int j = 0; j < RW; ++j) {
      const int c = rg + kDecGroups * j;
      const float kc = kt[c] * inv;
      float4 x = S[j];
      x.x = fmaf(alpha, x.x, coef.x * kc);
      x.y = fmaf(alpha, x.y, coef.y * kc);
      x.z = fmaf(alpha, x.z, coef.z * kc);
      x.w = fmaf(alpha, x.w, coef.w * kc);
      __stcs(reinterpret_cast<float4 *>(a.final_state + sbase + (int64_t)c * a.dv + r0), x);
    }
  }
  if (rg == 0 && active) {  // o = alpha p + coef (kt . q)
    p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < kDecGroups; ++r) {
      const float4 x = pq[r][cq];
      p.x += x.x;
      p.y += x.y;
      p.z += x.z;
      p.w += x.w;
    }
    const float ktq = kqt * inv;
    Tin *O = (Tin *)a.out + b * a.o_sb + t * a.o_st + h * a.o_sh + r0;
    O[0] = from_f32<Tin>(fmaf(alpha, p.x, coef.x * ktq));
    O[1] = from_f32<Tin>(fmaf(alpha, p.y, coef.y * ktq));
    O[2] = from_f32<Tin>(fmaf(alpha, p.z, coef.z * ktq));
    O[3] = from_f32<Tin>(fmaf(alpha, p.w, coef.w * ktq));
  }
}

template <typename Tin>
cudaError_t launch_decode(const DeltaArgs &a, cudaStream_t stream) {
  const int64_t grid = a.n_seqs * a.H * ((a.dv + kDecCols - 1) / kDecCols);
  if (grid == 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  switch (a.dk) {
    case 64: delta_decode_kernel<Tin, 64><<<(unsigned)grid, kDecThreads, 0, stream>>>(a); break;
    case 128: delta_decode_kernel<Tin, 128><<<(unsigned)grid, kDecThreads, 0, stream>>>(a); break;
    case 256: delta_decode_kernel<Tin, 256><<<(unsigned)grid, kDecThreads, 0, stream>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// One token per sequence: a dense batch with T = 1 (the host cannot see the
// lengths of a packed batch).
bool decode_shape(const DeltaArgs &a) {
  return !a.cu_seqlens && a.T == 1 && (a.dk == 64 || a.dk == 128 || a.dk == 256) && a.dv % 4 == 0 &&
         ((uintptr_t)a.init) % 16 == 0 && ((uintptr_t)a.final_state) % 16 == 0;
}

}  // namespace

cudaError_t launch_delta(const DeltaArgs &a, cudaStream_t stream) {
  if (decode_shape(a))
    return a.dtype == LA_F32 ? launch_decode<float>(a, stream) : launch_decode<__nv_bfloat16>(a, stream);
  return a.dtype == LA_F32 ? launch_dtype<float>(a, stream) : launch_dtype<__nv_bfloat16>(a, stream);
}

}  // namespace la
