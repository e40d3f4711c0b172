// la_ew.cu -- elementwise kernels: the steps of the backward pass outside the
// tensor-core passes, and the output RMSNorm with a Swish gate.
//
// The backward runs on the forward kernel (see la_bwd_chunk): with phi = elu + 1
// the operands that kernel reads untransformed must hold phi(x) already
// ("1.6 长上下文与高效注意力", section 线性注意力: phi(x) = elu(x) + 1), which
// phi_kernel writes in one pass over a [B, T, H, D] tensor (the passes' epilogues
// apply phi'); the per-token decay's log-decay gradient ends in a reverse
// cumulative sum per sequence and head.
#include <cuda_bf16.h>

#include "la_common.cuh"
#include "la_internal.h"

namespace la {
namespace {

constexpr int kEwThreads = 256;

// One thread per 16-byte vector of a row (VW elements; D is a multiple of VW):
// vector e is column block e mod (D / VW) of row e / (D / VW), rows ordered
// (b, t, h).
template <typename T>
struct Vec {
  static constexpr int VW = 16 / sizeof(T);
};

// Token row r of a [B, T, H] grid (rows ordered (b, t, h)) in the index type I:
// 32-bit whenever the launch's element count fits (the divisions are then a few
// instructions instead of a 64-bit division's long sequence).
template <typename I>
__device__ __forceinline__ void split_row(I row, I T_, I H, I &b, I &t, I &h) {
  h = row % H;
  const I bt = row / H;
  t = bt % T_;
  b = bt / T_;
}

template <typename T, typename I>
__global__ void __launch_bounds__(kEwThreads) phi_kernel(TensorView src, TensorView dst, I T_, I H, I D, I nvec,
                                                          int phi) {
  constexpr int VW = Vec<T>::VW;
  const I nvr = D / VW;
  for (I e = blockIdx.x * (I)kEwThreads + threadIdx.x; e < nvec; e += (I)gridDim.x * kEwThreads) {
    const I row = e / nvr;
    const int col = (int)(e - row * nvr) * VW;
    I b, t, h;
    split_row<I>(row, T_, H, b, t, h);
    const T *s = (const T *)src.data + (int64_t)b * src.sb + (int64_t)t * src.st + (int64_t)h * src.sh + col;
    T *o = (T *)dst.data + (int64_t)b * dst.sb + (int64_t)t * dst.st + (int64_t)h * dst.sh + col;
    uint4 x = *reinterpret_cast<const uint4 *>(s);
    T *xv = reinterpret_cast<T *>(&x);
#pragma unroll
    for (int u = 0; u < VW; ++u) xv[u] = from_f32<T>(feature_map(to_f32<T>(xv[u]), phi));
    *reinterpret_cast<uint4 *>(o) = x;
  }
}

__device__ __forceinline__ void unpack_bf16x8(const uint4 &u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float (&f)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 p = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t *>(&p);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Backward of the normalised forward (see la_bwd_chunk_norm).  With v' = [v, 1, 1, 0...]
// and u' = [u, e_hi, e_lo, 0...], u_t = dout_t / den_t and e_t = -(u_t . o_t) (the
// denominator's adjoint, o_t = num_t / den_t) split into a bf16 pair e_hi + e_lo,
// the unnormalised backward of (q, k, v', u') is the normalised one's.
//
// Rounding: the sums u_t . v_j + e_t that the backward forms cancel (for a one-token
// sequence exactly: o_1 = v_1 whatever q and k).  e_t is therefore taken from the
// bf16-rounded u_t, so that u' is the exact gradient for an output gradient within
// one bf16 rounding of dout, and carried to about 16 bits by the pair.
//
// Both kernels write contiguous [rows][dvp] bf16 rows, one thread per 16-byte
// vector (lpr = dvp / 8 vectors per row, a power of two, so a row's vectors sit
// in one warp); dv is a multiple of 8 below dvp.
template <typename T, typename I>
__global__ void __launch_bounds__(kEwThreads) aug_v_kernel(TensorView v, T *vp, I T_, I H, int dv, int lpr_log2,
                                                            I nvec) {
  constexpr int VW = Vec<T>::VW;
  const int lpr = 1 << lpr_log2;
  for (I e = blockIdx.x * (I)kEwThreads + threadIdx.x; e < nvec; e += (I)gridDim.x * kEwThreads) {
    const I row = e >> lpr_log2;
    const int col = (int)(e & (I)(lpr - 1)) * VW;
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (col < dv) {
      I b, t, h;
      split_row<I>(row, T_, H, b, t, h);
      x = *reinterpret_cast<const uint4 *>((const T *)v.data + (int64_t)b * v.sb + (int64_t)t * v.st +
                                           (int64_t)h * v.sh + col);
    } else if (col == dv) {  // ones in columns dv and dv + 1
      T *xv = reinterpret_cast<T *>(&x);
      xv[0] = xv[1] = from_f32<T>(1.f);
    }
    *reinterpret_cast<uint4 *>(vp + (int64_t)row * (VW << lpr_log2) + col) = x;
  }
}

// The CUDA-core route: rows of the unnormalised forward of (q, k, v'), [num, den,
// den, 0...], turned into [u, e_hi, e_lo, 0...] in place (e_t = -(u_t . num_t) /
// den_t from u_t as stored); dout through its strides; T is the rows' element type.
template <typename T, typename I>
__global__ void __launch_bounds__(kEwThreads) norm_grad_num_kernel(TensorView dout, T *up, I T_, I H, int dv,
                                                                    int lpr_log2, I nvec) {
  constexpr int VW = Vec<T>::VW;
  const int lpr = 1 << lpr_log2;
  const int lane = threadIdx.x & 31;
  const int den_lane = (lane & ~(lpr - 1)) + dv / VW;  // the lane of this row holding column dv
  for (I e0 = blockIdx.x * (I)kEwThreads; e0 < nvec; e0 += (I)gridDim.x * kEwThreads) {
    const I e = e0 + threadIdx.x;  // rows are whole within a warp and the loop bound is warp-uniform
    const bool live = e < nvec;
    const I row = live ? e >> lpr_log2 : 0;
    const int col = (int)(e & (I)(lpr - 1)) * VW;
    T *p = up + (int64_t)row * (VW << lpr_log2) + col;
    float f[VW], d[VW];
#pragma unroll
    for (int u = 0; u < VW; ++u) f[u] = d[u] = 0.f;
    if (live) {
      const uint4 x = *reinterpret_cast<const uint4 *>(p);
      const T *xv = reinterpret_cast<const T *>(&x);
#pragma unroll
      for (int u = 0; u < VW; ++u) f[u] = to_f32<T>(xv[u]);
      if (col < dv) {
        I b, t, h;
        split_row<I>(row, T_, H, b, t, h);
        const uint4 y = *reinterpret_cast<const uint4 *>((const T *)dout.data + (int64_t)b * dout.sb +
                                                         (int64_t)t * dout.st + (int64_t)h * dout.sh + col);
        const T *yv = reinterpret_cast<const T *>(&y);
#pragma unroll
        for (int u = 0; u < VW; ++u) d[u] = to_f32<T>(yv[u]);
      }
    }
    const float den = __shfl_sync(0xffffffffu, f[0], den_lane);
    const float inv = 1.f / den;
    float y[VW], dot = 0.f;
#pragma unroll
    for (int u = 0; u < VW; ++u) {
      y[u] = col < dv ? to_f32<T>(from_f32<T>(d[u] * inv)) : 0.f;  // u as stored
      dot = fmaf(y[u], f[u], dot);                                   // u . num
    }
    for (int s = lpr / 2; s > 0; s >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, s);
    if (!live) continue;
    if (col == dv) {
      const float ev = -dot * inv;
      y[0] = to_f32<T>(from_f32<T>(ev));
      y[1] = ev - y[0];
    }
    uint4 o;
    T *ov = reinterpret_cast<T *>(&o);
#pragma unroll
    for (int u = 0; u < VW; ++u) ov[u] = from_f32<T>(y[u]);
    *reinterpret_cast<uint4 *>(p) = o;
  }
}

// u' rows from the normalised forward's o ([rows][dv] bf16, contiguous) and den
// ([rows] fp32), and dout (through its strides); fp32 arithmetic.
template <typename I>
__global__ void __launch_bounds__(kEwThreads) norm_grad_out_kernel(TensorView dout, const __nv_bfloat16 *o,
                                                                    const float *den, __nv_bfloat16 *up, I T_, I H,
                                                                    int dv, int lpr_log2, I nvec) {
  const int lpr = 1 << lpr_log2;
  for (I e0 = blockIdx.x * (I)kEwThreads; e0 < nvec; e0 += (I)gridDim.x * kEwThreads) {
    const I e = e0 + threadIdx.x;  // rows are whole within a warp and the loop bound is warp-uniform
    const bool live = e < nvec;
    const I row = live ? e >> lpr_log2 : 0;
    const int col = (int)(e & (I)(lpr - 1)) * 8;
    float d[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float inv = 0.f;
    if (live && col < dv) {
      I b, t, h;
      split_row<I>(row, T_, H, b, t, h);
      unpack_bf16x8(*reinterpret_cast<const uint4 *>((const __nv_bfloat16 *)dout.data + (int64_t)b * dout.sb +
                                                      (int64_t)t * dout.st + (int64_t)h * dout.sh + col), d);
      unpack_bf16x8(*reinterpret_cast<const uint4 *>(o + (int64_t)row * dv + col), f);
    }
    if (live) inv = 1.f / den[row];
    float y[8], dot = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      y[u] = col < dv ? __bfloat162float(__float2bfloat16_rn(d[u] * inv)) : 0.f;  // u as stored
      dot = fmaf(y[u], f[u], dot);                               // u . o
    }
    for (int s = lpr / 2; s > 0; s >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, s);
    if (!live) continue;
    if (col == dv) {
      y[0] = __bfloat162float(__float2bfloat16_rn(-dot));
      y[1] = -dot - y[0];
    }
    *reinterpret_cast<uint4 *>(up + (int64_t)row * (8 << lpr_log2) + col) = pack_bf16x8(y);
  }
}

unsigned ew_grid(int64_t n) {
  const int64_t blocks = (n + kEwThreads - 1) / kEwThreads;
  return (unsigned)(blocks < 148 * 64 ? blocks : 148 * 64);
}

// 32-bit indices when every element index of a launch fits.
bool fits32(int64_t n) { return n < 0x7fffffffLL - 148 * 64 * kEwThreads; }

int log2_exact(int x) {
  int l = 0;
  while ((1 << l) < x) ++l;
  return (1 << l) == x ? l : -1;
}

// Gradient of the log decays (per-token decay backward).  With b the prefix sum of
// the log decays g, the loss sees b_s only through the weights exp(b_i - b_j) of
// o_i = sum_{j<=i} exp(b_i - b_j) (qh_i . kh_j) v_j, so dL/db_s = qh_s . dqh_s -
// kh_s . dkh_s and dg_t = sum_{s>=t} dL/db_s.  The backward passes' epilogues add
// the row terms into dg (chunk_tc_kernel); this kernel finishes the sum.
// dg_t <- sum_{s >= t} dg_s over each sequence, in place.  One CTA
// per (sequence, head) walks the sequence from its end in tiles of kEwThreads
// tokens: a block-wide inclusive scan in reversed order plus the running total.
__global__ void __launch_bounds__(kEwThreads) dg_rev_cumsum_kernel(float *dg, const int32_t *cu, int64_t T_,
                                                                    int64_t H) {
  __shared__ float wsum[kEwThreads / 32];
  const int64_t unit = blockIdx.x;
  const int64_t h = unit % H, n = unit / H;
  int64_t row0, len;  // token row of the sequence's first token in the [B * T] grid, and its length
  if (cu) {
    row0 = cu[n];
    len = (int64_t)cu[n + 1] - cu[n];
  } else {
    row0 = n * T_;
    len = T_;
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float carry = 0.f;
  for (int64_t k0 = 0; k0 < len; k0 += kEwThreads) {
    const int64_t k = k0 + tid;  // k-th token from the end
    const int64_t t = len - 1 - k;
    float x = k < len ? dg[(row0 + t) * H + h] : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    float before = carry;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    float tile = 0.f;
#pragma unroll
    for (int w = 0; w < kEwThreads / 32; ++w) tile += wsum[w];
    if (k < len) dg[(row0 + t) * H + h] = x + before;
    carry += tile;
    __syncthreads();  // wsum is rewritten by the next tile
  }
}


}  // namespace

// Both need 16-byte aligned rows (la_tensor's pointer and stride rules) and
// D a multiple of the vector width (every supported head dim is).
cudaError_t launch_phi_copy(TensorView src, TensorView dst, int64_t B, int64_t T, int64_t H, int64_t D, int phi,
                            int dtype, cudaStream_t stream) {
  const int vw = dtype == LA_F32 ? 4 : 8;
  if (D % vw) return cudaErrorInvalidValue;
  const int64_t n = B * T * H * (D / vw);
  if (n == 0) return cudaSuccess;
  const unsigned grid = ew_grid(n);
  if (fits32(n)) {
    const uint32_t T32 = (uint32_t)T, H32 = (uint32_t)H, D32 = (uint32_t)D, n32 = (uint32_t)n;
    if (dtype == LA_F32)
      phi_kernel<float, uint32_t><<<grid, kEwThreads, 0, stream>>>(src, dst, T32, H32, D32, n32, phi);
    else
      phi_kernel<__nv_bfloat16, uint32_t><<<grid, kEwThreads, 0, stream>>>(src, dst, T32, H32, D32, n32, phi);
  } else if (dtype == LA_F32) {
    phi_kernel<float, int64_t><<<grid, kEwThreads, 0, stream>>>(src, dst, T, H, D, n, phi);
  } else {
    phi_kernel<__nv_bfloat16, int64_t><<<grid, kEwThreads, 0, stream>>>(src, dst, T, H, D, n, phi);
  }
  return cudaGetLastError();
}

// dg_t <- sum_{s >= t} dg_s within each sequence (dense batch, or packed by cu_seqlens).
cudaError_t launch_dg_rev_cumsum(float *dg, const int32_t *cu_seqlens, int64_t n_seqs, int64_t T, int64_t H,
                                 cudaStream_t stream) {
  const int64_t units = n_seqs * H;
  if (units == 0 || T == 0) return cudaSuccess;
  if (units > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  dg_rev_cumsum_kernel<<<(unsigned)units, kEwThreads, 0, stream>>>(dg, cu_seqlens, T, H);
  return cudaGetLastError();
}

// v' = [v, 1, 1, 0...] into a contiguous [B * T * H][dvp] buffer of v's dtype (dv a
// multiple of the vector width below dvp, dvp / width a power of two up to 32).
cudaError_t launch_aug_v(TensorView v, void *vp, int64_t B, int64_t T, int64_t H, int dv, int dvp, int dtype,
                         cudaStream_t stream) {
  const int vw = dtype == LA_F32 ? 4 : 8;
  const int l = log2_exact(dvp / vw);
  if (dv % vw || dvp % vw || dvp <= dv || l < 0 || l > 5) return cudaErrorInvalidValue;
  const int64_t n = B * T * H * (dvp / vw);
  if (n == 0) return cudaSuccess;
  const unsigned grid = ew_grid(n);
  if (dtype == LA_F32) {
    float *out = static_cast<float *>(vp);
    if (fits32(n))
      aug_v_kernel<float, uint32_t><<<grid, kEwThreads, 0, stream>>>(v, out, (uint32_t)T, (uint32_t)H, dv, l,
                                                                      (uint32_t)n);
    else
      aug_v_kernel<float, int64_t><<<grid, kEwThreads, 0, stream>>>(v, out, T, H, dv, l, n);
  } else {
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(vp);
    if (fits32(n))
      aug_v_kernel<__nv_bfloat16, uint32_t><<<grid, kEwThreads, 0, stream>>>(v, out, (uint32_t)T, (uint32_t)H, dv,
                                                                              l, (uint32_t)n);
    else
      aug_v_kernel<__nv_bfloat16, int64_t><<<grid, kEwThreads, 0, stream>>>(v, out, T, H, dv, l, n);
  }
  return cudaGetLastError();
}

// [num, den, den, 0...] -> [u, e_hi, e_lo, 0...] in place (see norm_grad_num_kernel).
cudaError_t launch_norm_grad_num(TensorView dout, void *up, int64_t B, int64_t T, int64_t H, int dv, int dvp,
                                 int dtype, cudaStream_t stream) {
  const int vw = dtype == LA_F32 ? 4 : 8;
  const int l = log2_exact(dvp / vw);
  if (dv % vw || dvp % vw || dvp <= dv || l < 0 || l > 5) return cudaErrorInvalidValue;
  const int64_t n = B * T * H * (dvp / vw);
  if (n == 0) return cudaSuccess;
  const unsigned grid = ew_grid(n);
  if (dtype == LA_F32) {
    float *u = static_cast<float *>(up);
    if (fits32(n))
      norm_grad_num_kernel<float, uint32_t><<<grid, kEwThreads, 0, stream>>>(dout, u, (uint32_t)T, (uint32_t)H, dv,
                                                                              l, (uint32_t)n);
    else
      norm_grad_num_kernel<float, int64_t><<<grid, kEwThreads, 0, stream>>>(dout, u, T, H, dv, l, n);
  } else {
    __nv_bfloat16 *u = static_cast<__nv_bfloat16 *>(up);
    if (fits32(n))
      norm_grad_num_kernel<__nv_bfloat16, uint32_t><<<grid, kEwThreads, 0, stream>>>(
          dout, u, (uint32_t)T, (uint32_t)H, dv, l, (uint32_t)n);
    else
      norm_grad_num_kernel<__nv_bfloat16, int64_t><<<grid, kEwThreads, 0, stream>>>(dout, u, T, H, dv, l, n);
  }
  return cudaGetLastError();
}

// u' = [dout / den, e_hi, e_lo, 0...] per row from o, den and dout (see norm_grad_out_kernel).
cudaError_t launch_norm_grad_out(TensorView dout, const void *o, const float *den, void *up, int64_t B, int64_t T,
                                 int64_t H, int dv, int dvp, cudaStream_t stream) {
  const int l = log2_exact(dvp / 8);
  if (dv % 8 || dvp % 8 || dvp <= dv || l < 0 || l > 5) return cudaErrorInvalidValue;
  const int64_t n = B * T * H * (dvp / 8);
  if (n == 0) return cudaSuccess;
  const __nv_bfloat16 *ob = static_cast<const __nv_bfloat16 *>(o);
  __nv_bfloat16 *u = static_cast<__nv_bfloat16 *>(up);
  if (fits32(n))
    norm_grad_out_kernel<uint32_t><<<ew_grid(n), kEwThreads, 0, stream>>>(dout, ob, den, u, (uint32_t)T,
                                                                            (uint32_t)H, dv, l, (uint32_t)n);
  else
    norm_grad_out_kernel<int64_t><<<ew_grid(n), kEwThreads, 0, stream>>>(dout, ob, den, u, T, H, dv, l, n);
  return cudaGetLastError();
}

}  // namespace la

namespace la {
namespace {

// y = o / sqrt(mean(o^2) + eps) * w * g * sigmoid(g) over the d_v values of one
// (token, head): one warp per row, fp32 arithmetic, y may alias o.
template <typename T>
__global__ void __launch_bounds__(kEwThreads) norm_gate_kernel(TensorView o, TensorView g, TensorView y,
                                                                const float *w, float eps, int64_t T_,
                                                                int64_t H, int dv, int64_t rows) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (kEwThreads / 32);
  for (int64_t row = blockIdx.x * (int64_t)(kEwThreads / 32) + (threadIdx.x >> 5); row < rows; row += warps) {
    const int64_t h = row % H, t = (row / H) % T_, b = row / (H * T_);
    const T *op = (const T *)o.data + b * o.sb + t * o.st + h * o.sh;
    const T *gp = (const T *)g.data + b * g.sb + t * g.st + h * g.sh;
    T *yp = (T *)y.data + b * y.sb + t * y.st + h * y.sh;
    float ss = 0.f;
    for (int c = lane; c < dv; c += 32) {
      const float x = to_f32<T>(op[c]);
      ss = fmaf(x, x, ss);
    }
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, k);
    const float rstd = rsqrtf(ss / (float)dv + eps);
    for (int c = lane; c < dv; c += 32) {
      const float gv = to_f32<T>(gp[c]);
      yp[c] = from_f32<T>(to_f32<T>(op[c]) * rstd * w[c] * (gv / (1.f + expf(-gv))));
    }
  }
}

}  // namespace

cudaError_t launch_norm_gate(TensorView o, TensorView g, TensorView y, const float *w, float eps, int64_t B,
                             int64_t T, int64_t H, int dv, int dtype, cudaStream_t stream) {
  const int64_t rows = B * T * H;
  if (rows == 0) return cudaSuccess;
  const int64_t blocks = (rows + kEwThreads / 32 - 1) / (kEwThreads / 32);
  const unsigned grid = (unsigned)(blocks < 148 * 16 ? blocks : 148 * 16);
  if (dtype == LA_F32)
    norm_gate_kernel<float><<<grid, kEwThreads, 0, stream>>>(o, g, y, w, eps, T, H, dv, rows);
  else
    norm_gate_kernel<__nv_bfloat16><<<grid, kEwThreads, 0, stream>>>(o, g, y, w, eps, T, H, dv, rows);
  return cudaGetLastError();
}

}  // namespace la
