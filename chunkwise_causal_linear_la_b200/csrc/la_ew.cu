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

template <typename T>
__device__ __forceinline__ void row_of(int64_t e, int64_t nvr, int64_t T_, int64_t H, int64_t &b, int64_t &t,
                                       int64_t &h, int &col) {
  const int64_t row = e / nvr;
  col = (int)(e - row * nvr) * Vec<T>::VW;
  h = row % H;
  const int64_t bt = row / H;
  t = bt % T_;
  b = bt / T_;
}

template <typename T>
__global__ void __launch_bounds__(kEwThreads) phi_kernel(TensorView src, TensorView dst, int64_t T_, int64_t H,
                                                          int64_t D, int64_t nvec, int phi) {
  constexpr int VW = Vec<T>::VW;
  const int64_t nvr = D / VW;
  for (int64_t e = blockIdx.x * (int64_t)kEwThreads + threadIdx.x; e < nvec; e += (int64_t)gridDim.x * kEwThreads) {
    int64_t b, t, h;
    int col;
    row_of<T>(e, nvr, T_, H, b, t, h, col);
    const T *s = (const T *)src.data + b * src.sb + t * src.st + h * src.sh + col;
    T *o = (T *)dst.data + b * dst.sb + t * dst.st + h * dst.sh + col;
    uint4 x = *reinterpret_cast<const uint4 *>(s);
    T *xv = reinterpret_cast<T *>(&x);
#pragma unroll
    for (int u = 0; u < VW; ++u) xv[u] = from_f32<T>(feature_map(to_f32<T>(xv[u]), phi));
    *reinterpret_cast<uint4 *>(o) = x;
  }
}

// Gradient of the log decays (per-token decay backward).  With b the prefix sum of
// the log decays g, the loss sees b_s only through the weights exp(b_i - b_j) of
// o_i = sum_{j<=i} exp(b_i - b_j) (qh_i . kh_j) v_j, so dL/db_s = qh_s . dqh_s -
// kh_s . dkh_s and dg_t = sum_{s>=t} dL/db_s.  The backward passes' epilogues add
// the row terms into dg (chunk_tc_kernel); this kernel finishes the sum.
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
// the unnormalised forward returns [num, den, den, 0...] per row (den_t = sum_{j<=t}
// gamma^(t-j) phi(q_t) . phi(k_j) is a value column of ones), and with
// u' = [u, e_hi, e_lo, 0...], u_t = dout_t / den_t and e_t = -(u_t . num_t) / den_t
// (the denominator's adjoint) split into a bf16 pair e_hi + e_lo, the unnormalised
// backward of (q, k, v', u') is the normalised one's.
//
// Rounding: the sums u_t . v_j + e_t that the backward forms cancel (for a one-token
// sequence exactly: o_1 = v_1 whatever q and k).  e_t is therefore taken from the
// bf16-rounded u_t, so that u' is the exact gradient for an output gradient within
// one bf16 rounding of dout, and carried to about 16 bits by the pair.
//
// v' rows in a contiguous [rows][dvp] bf16 buffer: thread e writes the 16-byte
// vector e mod (dvp / 8) of row e / (dvp / 8); dv is a multiple of 8.
__global__ void __launch_bounds__(kEwThreads) aug_v_kernel(TensorView v, __nv_bfloat16 *vp, int64_t T_, int64_t H,
                                                            int dv, int dvp, int64_t nvec) {
  const int nvr = dvp / 8;
  for (int64_t e = blockIdx.x * (int64_t)kEwThreads + threadIdx.x; e < nvec; e += (int64_t)gridDim.x * kEwThreads) {
    const int64_t row = e / nvr;
    const int col = (int)(e - row * nvr) * 8;
    const int64_t h = row % H, bt = row / H, t = bt % T_, b = bt / T_;
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (col < dv)
      x = *reinterpret_cast<const uint4 *>((const __nv_bfloat16 *)v.data + b * v.sb + t * v.st + h * v.sh + col);
    else if (col == dv)
      x.x = 0x3F803F80u;  // bf16 1.0 in columns dv and dv + 1
    *reinterpret_cast<uint4 *>(vp + row * dvp + col) = x;
  }
}

// up rows ([rows][dvp] bf16): [num, den, den, 0...] in, [u, e_hi, e_lo, 0...] out
// (fp32 arithmetic), dout rows read through their strides.  lpr = dvp / 8 lanes per
// row, one vector each.
__global__ void __launch_bounds__(kEwThreads) norm_grad_out_kernel(TensorView dout, __nv_bfloat16 *up, int64_t T_,
                                                                    int64_t H, int dv, int dvp, int64_t rows) {
  const int lpr = dvp / 8;
  const int lane = threadIdx.x & 31, sub = lane % lpr;
  const int col = sub * 8;
  const int den_lane = (lane - sub) + dv / 8;  // the lane of this row holding column dv
  const int64_t rows_per_step = (int64_t)gridDim.x * (kEwThreads / lpr);
  for (int64_t row0 = blockIdx.x * (int64_t)(kEwThreads / lpr); row0 < rows; row0 += rows_per_step) {
    const int64_t row = row0 + threadIdx.x / lpr;
    const bool live = row < rows;
    float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, d[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    uint4 *p = reinterpret_cast<uint4 *>(up + (live ? row : 0) * dvp + col);
    if (live) {
      unpack_bf16x8(*p, f);
      if (col < dv) {
        const int64_t h = row % H, bt = row / H, t = bt % T_, b = bt / T_;
        unpack_bf16x8(*reinterpret_cast<const uint4 *>((const __nv_bfloat16 *)dout.data + b * dout.sb +
                                                        t * dout.st + h * dout.sh + col), d);
      }
    }
    const float den = __shfl_sync(0xffffffffu, f[0], den_lane);
    const float inv = 1.f / den;
    float y[8], dot = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      y[u] = col + u < dv ? __bfloat162float(__float2bfloat16_rn(d[u] * inv)) : 0.f;  // u as stored
      dot = fmaf(y[u], f[u], dot);  // u . num (zero past dv)
    }
    for (int o = lpr / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (!live) continue;
    if (col == dv) {
      const float e = -dot * inv;
      y[0] = __bfloat162float(__float2bfloat16_rn(e));
      y[1] = e - y[0];
    }
    *p = pack_bf16x8(y);
  }
}

unsigned ew_grid(int64_t n) {
  const int64_t blocks = (n + kEwThreads - 1) / kEwThreads;
  return (unsigned)(blocks < 148 * 16 ? blocks : 148 * 16);
}

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
  if (dtype == LA_F32)
    phi_kernel<float><<<ew_grid(n), kEwThreads, 0, stream>>>(src, dst, T, H, D, n, phi);
  else
    phi_kernel<__nv_bfloat16><<<ew_grid(n), kEwThreads, 0, stream>>>(src, dst, T, H, D, n, phi);
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

// v' = [v, 1, 1, 0...] into a contiguous [B * T * H][dvp] bf16 buffer (dv a multiple of 8, dvp > dv).
cudaError_t launch_aug_v(TensorView v, void *vp, int64_t B, int64_t T, int64_t H, int dv, int dvp,
                         cudaStream_t stream) {
  if (dv % 8 || dvp % 8 || dvp <= dv) return cudaErrorInvalidValue;
  const int64_t n = B * T * H * (dvp / 8);
  if (n == 0) return cudaSuccess;
  aug_v_kernel<<<ew_grid(n), kEwThreads, 0, stream>>>(v, static_cast<__nv_bfloat16 *>(vp), T, H, dv, dvp, n);
  return cudaGetLastError();
}

// [num, den, den, 0...] -> [u, e_hi, e_lo, 0...] in place, per row of up (see norm_grad_out_kernel).
cudaError_t launch_norm_grad_out(TensorView dout, void *up, int64_t B, int64_t T, int64_t H, int dv, int dvp,
                                 cudaStream_t stream) {
  const int lpr = dvp / 8;
  if (dv % 8 || dvp <= dv || lpr > 32 || (lpr & (lpr - 1))) return cudaErrorInvalidValue;
  const int64_t rows = B * T * H;
  if (rows == 0) return cudaSuccess;
  const int64_t blocks = (rows + kEwThreads / lpr - 1) / (kEwThreads / lpr);
  const unsigned grid = (unsigned)(blocks < 148 * 16 ? blocks : 148 * 16);
  norm_grad_out_kernel<<<grid, kEwThreads, 0, stream>>>(dout, static_cast<__nv_bfloat16 *>(up), T, H, dv, dvp, rows);
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
