// misc_kernels.cuh - the bandwidth-bound pieces of the TSP rank step and of
// the MLP-half backward: zigzag index map, pre-LayerNorm with fp16 output
// (one warp per row, or one block per row for wide rows), weight shard
// packing, the bf16 transposes and the LayerNorm backward of the backward
// pass, and the bounded-wait self test.
#pragma once
#include "ptx.cuh"

namespace tsp {

// Zigzag partition (TSP news item, zubnet.ai, paragraph 2): local token i of
// rank r sits at global position r*c + i (i < c) or (2D-1-r)*c + (i-c).
__global__ void zigzag_index_kernel(int32_t* idx, int64_t c, int D, int rank) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i >= 2 * c) return;
  idx[i] = static_cast<int32_t>(i < c ? rank * c + i : (2 * D - 1 - rank) * c + (i - c));
}

template <typename T>
__device__ __forceinline__ void load8(const T* src, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* src, float (&v)[8]) {
  const uint4 q = __ldg(reinterpret_cast<const uint4*>(src));
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
    v[2 * j] = f.x;
    v[2 * j + 1] = f.y;
  }
}

template <>
__device__ __forceinline__ void load8<__half>(const __half* src, float (&v)[8]) {
  const uint4 q = __ldg(reinterpret_cast<const uint4*>(src));
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
    v[2 * j] = f.x;
    v[2 * j + 1] = f.y;
  }
}

template <>
__device__ __forceinline__ void load8<float>(const float* src, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(src));
  const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// LayerNorm of one row per warp, gamma=1, beta=0:
//   y = (x - mean) / sqrt(var + eps), var biased, statistics in fp32 over the
//   row held in registers (two passes: mean, then centred sum of squares).
// Output fp16 (round to nearest even), the operand format of the matmul that
// follows.  MAXC = 8-element chunks per lane.
template <typename Tin, int MAXC>
__global__ void __launch_bounds__(256) layernorm_rows_kernel(const Tin* __restrict__ x, __half* __restrict__ y,
                                                             int64_t rows, int h, float eps) {
  const int warps = blockDim.x >> 5;
  const int64_t r = blockIdx.x * static_cast<int64_t>(warps) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const int nch = h >> 3;  // 8-element chunks in the row
  const Tin* xr = x + r * h;
  float v[MAXC][8];
  float sum = 0.f;
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int ch = lane + 32 * c;
    if (ch < nch) {
      load8<Tin>(xr + ch * 8, v[c]);
#pragma unroll
      for (int j = 0; j < 8; ++j) sum += v[c][j];
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[c][j] = 0.f;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum / h;
  float sq = 0.f;
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int ch = lane + 32 * c;
    if (ch < nch) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float d = v[c][j] - mean;
        sq = fmaf(d, d, sq);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const float rstd = rsqrtf(sq / h + eps);
  __half* yr = y + r * h;
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int ch = lane + 32 * c;
    if (ch < nch) {
      uint4 o;
      o.x = pack_half2((v[c][0] - mean) * rstd, (v[c][1] - mean) * rstd);
      o.y = pack_half2((v[c][2] - mean) * rstd, (v[c][3] - mean) * rstd);
      o.z = pack_half2((v[c][4] - mean) * rstd, (v[c][5] - mean) * rstd);
      o.w = pack_half2((v[c][6] - mean) * rstd, (v[c][7] - mean) * rstd);
      *reinterpret_cast<uint4*>(yr + ch * 8) = o;
    }
  }
}

// Shard packing: out[o][i] = w[(row0 + i) * ld + col0 + o] for o < n_out,
// i < n_in; i.e. a transposed sub-block of the math-orientation bf16 weight,
// converted to fp16 (round to nearest even, saturating) in the K-major
// [n_out, n_in] layout the GEMM's B operand uses.  32x32 tiles staged through
// shared memory so both sides are coalesced.
// A weight outside fp16's range sets kFlagFp16Saturated in status[1].
__global__ void pack_transpose_kernel(const __nv_bfloat16* __restrict__ w, int64_t ld, int64_t row0, int64_t col0,
                                      __half* __restrict__ out, int n_out, int n_in, int* status) {
  __shared__ float tile[32][33];
  const int i0 = blockIdx.x * 32, o0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  for (int k = ty; k < 32; k += 8) {
    const int i = i0 + k, o = o0 + tx;
    if (i < n_in && o < n_out) tile[k][tx] = __bfloat162float(w[(row0 + i) * ld + col0 + o]);
  }
  __syncthreads();
  float mx = 0.f;
  for (int k = ty; k < 32; k += 8) {
    const int o = o0 + k, i = i0 + tx;
    if (i < n_in && o < n_out) {
      uint16_t hbits;
      const float v = tile[tx][k];
      mx = fmaxf(mx, fabsf(v));
      asm("cvt.rn.satfinite.f16.f32 %0, %1;" : "=h"(hbits) : "f"(v));
      reinterpret_cast<uint16_t*>(out)[static_cast<int64_t>(o) * n_in + i] = hbits;
    }
  }
  note_fp16_saturation(status, mx);
}

// ---------------------------------------------------------------- backward helpers
template <typename T>
__device__ __forceinline__ void unpack8(uint4 v, float (&f)[8]);
template <>
__device__ __forceinline__ void unpack8<__half>(uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
    f[2 * j] = t.x;
    f[2 * j + 1] = t.y;
  }
}
template <>
__device__ __forceinline__ void unpack8<__nv_bfloat16>(uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
    f[2 * j] = t.x;
    f[2 * j + 1] = t.y;
  }
}

// out[c][r] = bf16(in[r][c]) for r < rows, c < cols (both multiples of 8):
// the K-major [cols, rows] operand of a weight-gradient matmul that reduces
// over the rows (tokens).  64 x 64 tiles staged through shared memory, read
// and written as 16-byte vectors of 8 elements.
template <typename Tin>
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const Tin* __restrict__ in, int64_t rows, int cols,
                                                             __nv_bfloat16* __restrict__ out) {
  __shared__ float tile[64][65];
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 64;
  const int c0 = blockIdx.y * 64;
  for (int q = threadIdx.x; q < 512; q += 256) {
    const int rr = q >> 3, cc = (q & 7) * 8;
    if (r0 + rr < rows && c0 + cc < cols) {
      float f[8];
      load8<Tin>(in + (r0 + rr) * cols + c0 + cc, f);
#pragma unroll
      for (int j = 0; j < 8; ++j) tile[rr][cc + j] = f[j];
    }
  }
  __syncthreads();
  for (int q = threadIdx.x; q < 512; q += 256) {
    const int cc = q >> 3, rr = (q & 7) * 8;
    if (c0 + cc < cols && r0 + rr < rows) {
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = pack_bf16x2(tile[rr + 2 * j][cc], tile[rr + 2 * j + 1][cc]);
      *reinterpret_cast<uint4*>(out + static_cast<int64_t>(c0 + cc) * rows + r0 + rr) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// Block-wide sum of `n` values per thread (n <= 2), 256 threads.
__device__ __forceinline__ void block_sum2(float& a, float& b, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) {
    red[2 * warp] = a;
    red[2 * warp + 1] = b;
  }
  __syncthreads();
  a = 0.f;
  b = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    a += red[2 * w];
    b += red[2 * w + 1];
  }
}

// LayerNorm forward for wide rows (h >= 1024), one row per 256-thread block:
// the same arithmetic as layernorm_rows_kernel (fp32 statistics over the row
// held in registers: mean, then the centred sum of squares; fp16 output,
// round to nearest even), with 4 G values per thread.  Small blocks with few
// registers keep many rows in flight per SM, which the one-warp-per-row
// kernel cannot at h = 4096.
template <typename Tin>
__device__ __forceinline__ void load4(const Tin* src, float* v);
template <>
__device__ __forceinline__ void load4<float>(const float* src, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(src);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* src, float* v) {
  const uint2 q = *reinterpret_cast<const uint2*>(src);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}

template <typename Tin, int G>
__global__ void __launch_bounds__(256) layernorm_block_kernel(const Tin* __restrict__ x, __half* __restrict__ y, int h,
                                                              float eps) {
  __shared__ float red[16];
  const int64_t row = blockIdx.x;
  const Tin* xr = x + row * h;
  float v[4 * G];
  float sum = 0.f, dummy = 0.f;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int col = (g * 256 + threadIdx.x) * 4;
    if (col < h) {
      load4<Tin>(xr + col, &v[4 * g]);
      sum += (v[4 * g] + v[4 * g + 1]) + (v[4 * g + 2] + v[4 * g + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) v[4 * g + j] = 0.f;
    }
  }
  block_sum2(sum, dummy, red);
  const float mean = sum / h;
  float sq = 0.f;
  dummy = 0.f;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int col = (g * 256 + threadIdx.x) * 4;
    if (col < h) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float d = v[4 * g + j] - mean;
        sq = fmaf(d, d, sq);
      }
    }
  }
  block_sum2(sq, dummy, red);
  const float rstd = rsqrtf(sq / h + eps);
  __half* yr = y + row * h;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int col = (g * 256 + threadIdx.x) * 4;
    if (col < h)
      *reinterpret_cast<uint2*>(yr + col) =
          make_uint2(pack_half2((v[4 * g] - mean) * rstd, (v[4 * g + 1] - mean) * rstd),
                     pack_half2((v[4 * g + 2] - mean) * rstd, (v[4 * g + 3] - mean) * rstd));
  }
}

// LayerNorm backward with the residual, one row per 256-thread block:
//   dy1 = dy + rstd * (g - mean(g) - xhat * mean(g * xhat)),
//   xhat = (y1 - mean(y1)) * rstd, rstd = 1 / sqrt(var(y1) + eps)
// (biased variance, gamma = 1, beta = 0), statistics in fp32 from the row
// held in registers (VPT values per thread, as groups of 4).  y1 (the
// LayerNorm's input) is fp32 or bf16, dy (the residual's gradient) bf16 or
// fp32; dy1 may be dy itself (each value is read before it is written).
// dy1_bf16, when not null, receives a bf16 copy of dy1.
template <typename Tx, typename Tr>
__device__ __forceinline__ void load4f(const Tx* src, float* v);
template <>
__device__ __forceinline__ void load4f<float, float>(const float* src, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(src);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <>
__device__ __forceinline__ void load4f<__nv_bfloat16, __nv_bfloat16>(const __nv_bfloat16* src, float* v) {
  const uint2 q = *reinterpret_cast<const uint2*>(src);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}

template <int VPT, typename Tx, typename Tr>
__global__ void __launch_bounds__(256) ln_backward_rows_kernel(const Tx* __restrict__ y1,
                                                               const float* __restrict__ g, const Tr* dy,
                                                               float* dy1, __nv_bfloat16* __restrict__ dy1_bf16,
                                                               int h, float eps) {
  __shared__ float red[16];
  const int64_t row = blockIdx.x;
  const Tx* yr = y1 + row * h;
  const float* gr = g + row * h;
  float yv[VPT], gv[VPT];
  float sum = 0.f, dummy = 0.f;
#pragma unroll
  for (int i = 0; i < VPT / 4; ++i) {
    const int col = (i * 256 + threadIdx.x) * 4;
    if (col < h) {
      load4f<Tx, Tx>(yr + col, &yv[4 * i]);
      const float4 b = *reinterpret_cast<const float4*>(gr + col);
      gv[4 * i] = b.x; gv[4 * i + 1] = b.y; gv[4 * i + 2] = b.z; gv[4 * i + 3] = b.w;
      sum += (yv[4 * i] + yv[4 * i + 1]) + (yv[4 * i + 2] + yv[4 * i + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) yv[4 * i + j] = gv[4 * i + j] = 0.f;
    }
  }
  block_sum2(sum, dummy, red);
  const float mean = sum / h;
  float sq = 0.f;
  dummy = 0.f;
#pragma unroll
  for (int i = 0; i < VPT / 4; ++i) {
    const int col = (i * 256 + threadIdx.x) * 4;
    if (col < h) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float d = yv[4 * i + j] - mean;
        sq = fmaf(d, d, sq);
      }
    }
  }
  block_sum2(sq, dummy, red);
  const float rstd = rsqrtf(sq / h + eps);
  float sg = 0.f, sgx = 0.f;
#pragma unroll
  for (int i = 0; i < VPT / 4; ++i) {
    const int col = (i * 256 + threadIdx.x) * 4;
    if (col < h) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        yv[4 * i + j] = (yv[4 * i + j] - mean) * rstd;  // xhat
        sg += gv[4 * i + j];
        sgx = fmaf(gv[4 * i + j], yv[4 * i + j], sgx);
      }
    }
  }
  block_sum2(sg, sgx, red);
  const float mg = sg / h, mgx = sgx / h;
  const Tr* dr = dy + row * h;
  float* outr = dy1 + row * h;
#pragma unroll
  for (int i = 0; i < VPT / 4; ++i) {
    const int col = (i * 256 + threadIdx.x) * 4;
    if (col < h) {
      float d[4];
      load4f<Tr, Tr>(dr + col, d);
      float4 o;
      o.x = d[0] + rstd * (gv[4 * i] - mg - yv[4 * i] * mgx);
      o.y = d[1] + rstd * (gv[4 * i + 1] - mg - yv[4 * i + 1] * mgx);
      o.z = d[2] + rstd * (gv[4 * i + 2] - mg - yv[4 * i + 2] * mgx);
      o.w = d[3] + rstd * (gv[4 * i + 3] - mg - yv[4 * i + 3] * mgx);
      *reinterpret_cast<float4*>(outr + col) = o;
      if (dy1_bf16)
        *reinterpret_cast<uint2*>(dy1_bf16 + row * h + col) = make_uint2(pack_bf16x2(o.x, o.y), pack_bf16x2(o.z, o.w));
    }
  }
}

// out = bf16(in), n a multiple of 8 (row-major copies of fp32 gradients for
// the bf16 tensor-core products).
__global__ void __launch_bounds__(256) convert_bf16_kernel(const float* __restrict__ in, __nv_bfloat16* __restrict__ out,
                                                           int64_t n) {
  const int64_t i = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) * 8;
  if (i >= n) return;
  const float4 a = *reinterpret_cast<const float4*>(in + i);
  const float4 b = *reinterpret_cast<const float4*>(in + i + 4);
  *reinterpret_cast<uint4*>(out + i) =
      make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
}

// The key owner's rows of the summed dK, dV after the reduce-scatter: for
// local row i at global position pos(i) (the zigzag map: r*c + i for i < c,
// (2D-1-r)*c + (i-c) after), out[i] = [bf16(dk[pos(i)]) | bf16(dv[pos(i)])],
// an [L, 2h] row-major bf16 matrix.  One thread per 8 columns.
__global__ void __launch_bounds__(256) gather_kv_grad_kernel(const float* __restrict__ dk, const float* __restrict__ dv,
                                                             __nv_bfloat16* __restrict__ out, int64_t L, int h,
                                                             int64_t c, int64_t off0, int64_t off1) {
  const int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int per_row = (2 * h) / 8;
  const int64_t i = t / per_row;
  if (i >= L) return;
  const int col = static_cast<int>(t - i * per_row) * 8;
  const int64_t pos = i < c ? off0 + i : off1 + i;
  const float* src = (col < h ? dk + pos * h + col : dv + pos * h + (col - h));
  const float4 a = *reinterpret_cast<const float4*>(src);
  const float4 b = *reinterpret_cast<const float4*>(src + 4);
  *reinterpret_cast<uint4*>(out + i * 2 * h + col) =
      make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
}

// The all-reduce of a tensor-parallel layer, on one GPU: out = resid +
// sum_k part[k] over the n_parts fp32 partial products [n] (each rank's
// row-parallel product), with the residual bf16 or fp32 and the output fp32
// or bf16.  Four values per thread; n a multiple of 4.
struct PartList {
  const float* p[16];
};

template <typename Tr, bool kOutF32>
__global__ void __launch_bounds__(256) sum_partials_kernel(PartList parts, int n_parts, const Tr* __restrict__ resid,
                                                           void* __restrict__ out, int64_t n) {
  const int64_t i = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) * 4;
  if (i >= n) return;
  float v[4];
  load4f<Tr, Tr>(resid + i, v);
  for (int k = 0; k < n_parts; ++k) {
    const float4 a = *reinterpret_cast<const float4*>(parts.p[k] + i);
    v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
  }
  if (kOutF32)
    *reinterpret_cast<float4*>(static_cast<float*>(out) + i) = make_float4(v[0], v[1], v[2], v[3]);
  else
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out) + i) =
        make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}

// Self test of the bounded waits: one thread waits on a barrier that expects
// an arrival nobody makes.  The wait gives up after timeout_ns, records the
// timeout in the status word and the kernel returns normally.
__global__ void wait_timeout_selftest_kernel(int* status, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl ctl{&abort_flag, status, timeout_ns};
    mbar_wait(&bar, 0, ctl);
  }
}

}  // namespace tsp
