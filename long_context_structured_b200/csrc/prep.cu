// prep.cu -- K1: rotary table and the elementwise prep pass.
//
// Rotary convention: rotate-half; pair (c, c + d/2) turns by the angle
// p * s * theta^(-2c/d), s the position-interpolation scale (1 = none).  The capped logit ("LM-Infinite", section 方法, RoPE
// realisation of d'_ij = min(d_ij, L)) needs, besides R(i) q_i and R(j) k_j,
// the query rotated to the cap, R(L) q_i, paired with the unrotated key.
//
// Outputs (all optional): Qr = R(i) q_i, Qc = R(L) q_i, Kr = R(j) k_j as bf16
// tensor-core operands; the fp32 logits of the starting-span ("sink") keys,
// computed from fp32 rotations of the exact inputs so that the large sink
// logits do not inherit bf16 operand rounding; and per (batch, kv head) the
// largest key norm, used by the top-k selector to bound bf16 scoring error.
//
// Work layout (HBM-bound): a thread owns 8 consecutive rotary pairs of one
// position -- one 16-byte load from each half of the query row (and of the
// key row at the same position, when the block's head is also a kv head),
// four 16-byte table loads shared by both rows, two 16-byte stores per row --
// so d/16 threads cover a position (8 for d = 128).  Each thread issues the
// loads of two positions before it computes either, which keeps enough bytes
// in flight per SM to cover HBM latency.  A block walks kRowsPerBlock
// positions of one head; the sink keys of that head's kv head are staged once
// per block in shared memory (rotated to their own position, and in the
// capped form R(-L) k used with the unrotated query).
#include <cmath>

#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"
#include "simt.cuh"
#include "status.cuh"

namespace sattn {

namespace {

constexpr int kPrepThreads = 256;
constexpr int kRowsPerBlock = 128;
constexpr int kU = 2;  // rows per thread whose loads are in flight together
constexpr int kMaxSmemSinks = 16;
constexpr int kPairsPerThread = 8;

// theta^(-2c/d) for the d/2 rotary pairs, computed once on the host in
// double and passed by value
struct InvFreq {
  double v[64];
};

// rows [0, n_low) and [row_lo, npos) of the table (the rows between are
// left as they are); I is the index type (32 bits whenever the entries fit)
template <typename I>
__global__ void rope_table_kernel(float2* tab, int npos, int half, const InvFreq inv_freq, double scale, int n_low,
                                  int row_lo) {
  const I n = (I)(n_low + (npos - row_lo)) * (I)half;
  for (I x = (I)blockIdx.x * blockDim.x + threadIdx.x; x < n; x += (I)gridDim.x * blockDim.x) {
    const int q = (int)(x / (I)half);
    const int c = (int)(x - (I)q * (I)half);
    const int p = q < n_low ? q : row_lo + (q - n_low);
    // the angle in double, reduced by whole turns in double (exact to
    // ~1e-12 for the positions used), then the fp32 sine and cosine of the
    // reduced angle: within a few fp32 ulps of the double-precision values
    const double ang = (double)p * scale * inv_freq.v[c];
    const double turns = rint(ang * (1.0 / 6.283185307179586));
    const float r = (float)fma(-turns, 6.283185307179586, ang);
    float s, co;
    sincosf(r, &s, &co);
    tab[(size_t)p * half + c] = make_float2(co, s);
  }
}

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 v = __bfloat1622float2(h[e]);
    f[2 * e] = v.x;
    f[2 * e + 1] = v.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
  return u;
}

// cos/sin of 8 consecutive pairs as four raw float4 loads (identity without a table)
__device__ __forceinline__ void load_tab8_raw(const float2* tab, int64_t pos, int half, int c0, float4* t) {
  if (!tab) {
#pragma unroll
    for (int e = 0; e < 4; ++e) t[e] = make_float4(1.f, 0.f, 1.f, 0.f);
    return;
  }
  const float4* src = reinterpret_cast<const float4*>(tab + pos * half + c0);
#pragma unroll
  for (int e = 0; e < 4; ++e) t[e] = src[e];
}

// (x0, x1) -> R x for 8 pairs with the cos/sin of load_tab8_raw
__device__ __forceinline__ void rotate8(const float* x0, const float* x1, const float4* t, float* r0, float* r1) {
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float c_a = t[e].x, s_a = t[e].y, c_b = t[e].z, s_b = t[e].w;
    r0[2 * e] = x0[2 * e] * c_a - x1[2 * e] * s_a;
    r1[2 * e] = x1[2 * e] * c_a + x0[2 * e] * s_a;
    r0[2 * e + 1] = x0[2 * e + 1] * c_b - x1[2 * e + 1] * s_b;
    r1[2 * e + 1] = x1[2 * e + 1] * c_b + x0[2 * e + 1] * s_b;
  }
}

// ALiBi bias of pair (i, j) in units of the unscaled logit q.k (0 without ALiBi)
__device__ __forceinline__ float alibi_bias_qk(const PrepArgs& a, int h, int i, int j) {
  if (!a.alibi) return 0.f;
  const int dist = (a.L > 0) ? min(i - j, a.L) : (i - j);
  return alibi_slope_qk(h, a.Hq, a.d) * (float)dist;
}

// Shared-memory slot of element c (< d/2) of a staged sink-key half: the 8
// elements c0..c0+7 of thread `sub` = c / 8 sit as two float4 at
// q * 4 * TPR + sub * 4 (q = 0, 1), so the TPR threads of a row read 64
// contiguous bytes per 16-byte load (no bank conflicts).
template <int TPR>
__device__ __forceinline__ int sink_slot(int c) {
  return ((c & 7) >> 2) * (4 * TPR) + (c >> 3) * 4 + (c & 3);
}

// <(u0, u1), (k0, k1)> over this thread's 8 pairs, k read from a staged row
template <int TPR>
__device__ __forceinline__ float sink_dot(const float* u0, const float* u1, const float* kv, int sub) {
  constexpr int half = TPR * 8;
  const float4 a = *reinterpret_cast<const float4*>(kv + sub * 4);
  const float4 b = *reinterpret_cast<const float4*>(kv + 4 * TPR + sub * 4);
  const float4 c = *reinterpret_cast<const float4*>(kv + half + sub * 4);
  const float4 e = *reinterpret_cast<const float4*>(kv + half + 4 * TPR + sub * 4);
  float A0 = 0.f, A1 = 0.f;
  fma2(A0, A1, u0[0], u0[1], a.x, a.y, A0, A1);
  fma2(A0, A1, u0[2], u0[3], a.z, a.w, A0, A1);
  fma2(A0, A1, u0[4], u0[5], b.x, b.y, A0, A1);
  fma2(A0, A1, u0[6], u0[7], b.z, b.w, A0, A1);
  fma2(A0, A1, u1[0], u1[1], c.x, c.y, A0, A1);
  fma2(A0, A1, u1[2], u1[3], c.z, c.w, A0, A1);
  fma2(A0, A1, u1[4], u1[5], e.x, e.y, A0, A1);
  fma2(A0, A1, u1[6], u1[7], e.z, e.w, A0, A1);
  return A0 + A1;
}

// grid (ceil(T / kRowsPerBlock), Hq, B).  Block (x, h, b) handles positions
// [x * kRowsPerBlock, ...) of query head h and, when h < Hkv, the key rows of
// kv head h at the same positions, so one table load serves both rows.  Each
// thread issues the loads of kU rows before it uses any of them.
// NSP: 0 = no sink logits; 4, 8, 16 = sink keys staged in shared memory
// (NSP >= n_sink slots); -1 = more sinks than that, read from global memory.
template <int D, int NSP>
__global__ void __launch_bounds__(kPrepThreads, 2) prep_kernel(PrepArgs a) {
  constexpr int half = D / 2;
  constexpr int tpr = half / kPairsPerThread;  // threads per row: 8 (d=128) or 4 (d=64)
  constexpr int rows_per_step = kPrepThreads / tpr;
  constexpr int NS_SMEM = NSP > 0 ? NSP : 1;
  __shared__ __align__(16) float s_sink_cap[NS_SMEM][D];  // R(-L) k_j: dotted with the raw query
  __shared__ __align__(16) float s_sink_rot[NS_SMEM][D];  // R(j) k_j: dotted with R(i) q_i
  __shared__ __align__(16) float s_lc[half];
  __shared__ __align__(16) float s_ls[half];  // cos/sin of the rotation to the cap L
  if (a.status && status_failed(a.status)) return;
  const int sub = threadIdx.x % tpr;       // which 8-pair chunk of the row
  const int c0 = sub * kPairsPerThread;
  const int b = blockIdx.z;
  const int h = blockIdx.y;
  const int g = h / (a.Hq / a.Hkv);
  const bool do_k = h < a.Hkv && (a.Kr != nullptr || a.kmax != nullptr);
  const int row_begin = blockIdx.x * kRowsPerBlock;
  const int row_end = min(a.T, row_begin + kRowsPerBlock);
  const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.Q) + b * a.q_sb + h * a.q_sh;
  const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(a.K);
  const __nv_bfloat16* Kh = K + b * a.k_sb + h * a.k_sh;
  // lanes of this thread's row group (8 or 4 consecutive lanes)
  const unsigned grp_mask = (tpr == 8) ? (0xffu << (threadIdx.x & 24)) : (0xfu << (threadIdx.x & 28));
  const int n_sink = NSP != 0 ? a.n_sink : 0;

  for (int c = threadIdx.x; c < half; c += kPrepThreads) {
    const float2 t = (a.L > 0 && a.tab) ? a.tab[(int64_t)a.L * half + c] : make_float2(1.f, 0.f);
    s_lc[c] = t.x;
    s_ls[c] = t.y;
  }
  if (NSP > 0) {
    __syncthreads();
    for (int x = threadIdx.x; x < n_sink * half; x += kPrepThreads) {
      const int j = x / half, c = x % half;
      const __nv_bfloat16* kp = K + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st;
      const float k0 = __bfloat162float(kp[c]), k1 = __bfloat162float(kp[c + half]);
      const float2 t = a.tab ? a.tab[(int64_t)j * half + c] : make_float2(1.f, 0.f);
      const int sl = sink_slot<tpr>(c);
      // <R(L) q, k> = <q, R(-L) k>: the capped logit of a sink key as a dot
      // product with the unrotated query
      s_sink_cap[j][sl] = k0 * s_lc[c] + k1 * s_ls[c];
      s_sink_cap[j][half + sl] = k1 * s_lc[c] - k0 * s_ls[c];
      s_sink_rot[j][sl] = k0 * t.x - k1 * t.y;
      s_sink_rot[j][half + sl] = k1 * t.x + k0 * t.y;
    }
  }
  __syncthreads();

  float kmax_sq = 0.f;
  for (int base = row_begin; base < row_end; base += rows_per_step * kU) {
    int ii[kU];
    bool ok[kU];
    uint4 qa[kU], qb[kU], ka[kU], kb[kU];
    float4 t[kU][4];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      ii[u] = base + u * rows_per_step + (int)threadIdx.x / tpr;
      ok[u] = ii[u] < row_end;
      if (ok[u]) {
        const __nv_bfloat16* qp = Q + (int64_t)ii[u] * a.q_st;
        qa[u] = *reinterpret_cast<const uint4*>(qp + c0);
        qb[u] = *reinterpret_cast<const uint4*>(qp + c0 + half);
        load_tab8_raw(a.tab, (int64_t)ii[u] + a.pos0, half, c0, t[u]);
        if (do_k) {
          const __nv_bfloat16* kp = Kh + (int64_t)ii[u] * a.k_st;
          ka[u] = *reinterpret_cast<const uint4*>(kp + c0);
          kb[u] = *reinterpret_cast<const uint4*>(kp + c0 + half);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (!ok[u]) continue;  // uniform over the row group
      const int i = ii[u];
      // ---- key row j = i of kv head h ----
      if (do_k) {
        float k0[8], k1[8];
        unpack8(ka[u], k0);
        unpack8(kb[u], k1);
        if (a.Kr) {
          float r0[8], r1[8];
          rotate8(k0, k1, t[u], r0, r1);
          __nv_bfloat16* kr =
              a.Kr + (((int64_t)b * a.Hkv + h) * (a.kr_rows > 0 ? a.kr_rows : a.T) + a.kr_row0 + i) * D;
          *reinterpret_cast<uint4*>(kr + c0) = pack8(r0);
          *reinterpret_cast<uint4*>(kr + c0 + half) = pack8(r1);
        }
        if (a.kmax) {
          float ss = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) ss = fmaf(k0[e], k0[e], fmaf(k1[e], k1[e], ss));
          for (int o = tpr / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(grp_mask, ss, o);
          kmax_sq = fmaxf(kmax_sq, ss);  // squared norm of key row i
        }
      }
      // ---- query row i of head h ----
      float x0[8], x1[8], r0[8], r1[8];
      unpack8(qa[u], x0);
      unpack8(qb[u], x1);
      rotate8(x0, x1, t[u], r0, r1);
      const int64_t orow = (((int64_t)b * a.Hq + h) * a.T + i) * D;
      if (a.Qr) {
        *reinterpret_cast<uint4*>(a.Qr + orow + c0) = pack8(r0);
        *reinterpret_cast<uint4*>(a.Qr + orow + c0 + half) = pack8(r1);
      }
      if (a.Qc) {
        float q0[8], q1[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          q0[e] = x0[e] * s_lc[c0 + e] - x1[e] * s_ls[c0 + e];
          q1[e] = x1[e] * s_lc[c0 + e] + x0[e] * s_ls[c0 + e];
        }
        *reinterpret_cast<uint4*>(a.Qc + orow + c0) = pack8(q0);
        *reinterpret_cast<uint4*>(a.Qc + orow + c0 + half) = pack8(q1);
      }
      const int64_t zrow = (((int64_t)b * a.Hq + h) * a.T + i) * n_sink;
      if (NSP > 0) {
        // sink logit j: capped (i - j > L): <q, R(-L) k_j> with the raw
        // query; otherwise <R(i) q, R(j) k_j>
        float z[NS_SMEM];
#pragma unroll
        for (int j = 0; j < NS_SMEM; ++j) {
          z[j] = 0.f;
          if (j < n_sink) {
            if (a.L > 0 && (i - j) > a.L) z[j] = sink_dot<tpr>(x0, x1, s_sink_cap[j], sub);
            else z[j] = sink_dot<tpr>(r0, r1, s_sink_rot[j], sub);
          }
        }
        group_reduce_transposed<NS_SMEM, tpr>(z, grp_mask, (int)threadIdx.x);
        constexpr int per = NS_SMEM >= tpr ? NS_SMEM / tpr : 1;
        constexpr int dup = NS_SMEM >= tpr ? 1 : tpr / NS_SMEM;
        if (sub % dup == 0) {
#pragma unroll
          for (int q = 0; q < per; ++q) {
            const int j = (sub / dup) * per + q;
            if (j < n_sink) a.sink_z[zrow + j] = (j <= i) ? z[q] - alibi_bias_qk(a, h, i, j) : -CUDART_INF_F;
          }
        }
      } else if (NSP < 0) {
        for (int j = 0; j < n_sink; ++j) {
          // every thread of a row group takes the same branch (same i and j)
          float z = -CUDART_INF_F;
          if (j <= i) {
            const bool capped = a.L > 0 && (i - j) > a.L;
            const __nv_bfloat16* kp = K + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st;
            float k0[8], k1[8];
            unpack8(*reinterpret_cast<const uint4*>(kp + c0), k0);
            unpack8(*reinterpret_cast<const uint4*>(kp + c0 + half), k1);
            float acc = 0.f;
            if (capped) {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float kc0 = k0[e] * s_lc[c0 + e] + k1[e] * s_ls[c0 + e];
                const float kc1 = k1[e] * s_lc[c0 + e] - k0[e] * s_ls[c0 + e];
                acc = fmaf(x0[e], kc0, fmaf(x1[e], kc1, acc));
              }
            } else {
              float4 tk[4];
              float kr0[8], kr1[8];
              load_tab8_raw(a.tab, j, half, c0, tk);
              rotate8(k0, k1, tk, kr0, kr1);
#pragma unroll
              for (int e = 0; e < 8; ++e) acc = fmaf(r0[e], kr0[e], fmaf(r1[e], kr1[e], acc));
            }
            for (int o = tpr / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(grp_mask, acc, o);
            z = acc;
          }
          if (sub == (j % tpr)) a.sink_z[zrow + j] = (j <= i) ? z - alibi_bias_qk(a, h, i, j) : z;
        }
      }
    }
  }
  if (do_k && a.kmax) {
    float v = kmax_sq;
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0) atomicMax(a.kmax + (size_t)b * a.Hkv + h, __float_as_uint(sqrtf(v)));
  }
}

}  // namespace

cudaError_t launch_rope_table_rows(float2* tab, int npos, int d, double theta, double scale, int n_low, int row_lo,
                                   cudaStream_t st) {
  const int half = d / 2;
  row_lo = std::max(0, std::min(row_lo, npos));
  n_low = std::max(0, std::min(n_low, row_lo));
  const int64_t n = ((int64_t)n_low + (npos - row_lo)) * half;
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>((n + threads - 1) / threads, 148 * 4);
  if (half > 64) return cudaErrorInvalidValue;
  InvFreq inv{};
  for (int c = 0; c < half; ++c) inv.v[c] = std::pow(theta, -2.0 * (double)c / (double)d);
  if (n + blocks * threads < ((int64_t)1 << 32))
    rope_table_kernel<uint32_t><<<(unsigned)blocks, threads, 0, st>>>(tab, npos, half, inv, scale, n_low, row_lo);
  else
    rope_table_kernel<uint64_t><<<(unsigned)blocks, threads, 0, st>>>(tab, npos, half, inv, scale, n_low, row_lo);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(float2* tab, int npos, int d, double theta, double scale, cudaStream_t st) {
  return launch_rope_table_rows(tab, npos, d, theta, scale, 0, 0, st);
}

template <int D>
cudaError_t launch_prep_d(const PrepArgs& a, cudaStream_t st) {
  dim3 grid((a.T + kRowsPerBlock - 1) / kRowsPerBlock, a.Hq, a.B);
  const int ns = a.sink_z ? a.n_sink : 0;
  if (ns == 0) prep_kernel<D, 0><<<grid, kPrepThreads, 0, st>>>(a);
  else if (ns <= 4) prep_kernel<D, 4><<<grid, kPrepThreads, 0, st>>>(a);
  else if (ns <= 8) prep_kernel<D, 8><<<grid, kPrepThreads, 0, st>>>(a);
  else if (ns <= kMaxSmemSinks) prep_kernel<D, kMaxSmemSinks><<<grid, kPrepThreads, 0, st>>>(a);
  else prep_kernel<D, -1><<<grid, kPrepThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_prep(const PrepArgs& a, cudaStream_t st) {
  if (a.f32) return cudaErrorInvalidValue;  // the fp32 path rotates inside its own kernel
  if (a.pos0 != 0 && a.sink_z) return cudaErrorInvalidValue;  // sink logits assume row = position
  if (a.B == 0 || a.T == 0) return cudaSuccess;
  if (a.d == 128) return launch_prep_d<128>(a, st);
  if (a.d == 64) return launch_prep_d<64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace sattn
