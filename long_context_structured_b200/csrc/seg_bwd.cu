// seg_bwd.cu -- backward pass of segmented execution ("Training-Inference
// Consistent Segmented Execution for Long-Context LLMs", sections 整体框架 and
// 损失函数 / 训练策略: training runs segment by segment), on the CUDA cores.
//
// The key list of a row i of segment s (as in the forward):
//   local heads: the keys [max(0, sS - M), i] at their global positions (the
//     carried tail and the segment, a pure shift of the re-based positions);
//   long heads: the cnt retrieved keys of the segment's prefix, key
//     blk_id * blk + o of prefix slot p = q * blk + o at the virtual position
//     sS - cnt + p, then the segment's keys [sS, i] at global positions.
// The query sits at its global position i, so every logit has the re-based
// distance.  The retrieved blocks are constants of the backward pass, as the
// top-k sets are: a retrieved key's gradient returns to its source position
// through the rotary position it had in the prefix, and a key used by
// several rows, heads or segments sums their contributions.  With
// P = exp(z / sqrt(d) - LSE_i), D_i = dO_i . O_i and dz = P (dO_i . v_j - D_i)
// / sqrt(d):  dq_i += R(i)^T dz R(pos_j) k_j,  dk_j += R(pos_j)^T dz R(i) q_i,
// dv_j += P dO_i.
//
//   seg_bwd_rows_kernel   a warp per query row: D_i and dq_i;
//   seg_bwd_keys_kernel   a warp per key: dk_j, dv_j over every row that
//                         keeps the key, in a fixed order (kv group's heads
//                         ascending; per head the key's own and later
//                         segments ascending, rows ascending; then, for the
//                         long heads, the segments whose prefix retrieved
//                         it, ascending).
// No atomics: bit for bit identical on repeat.
#include <math_constants.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float warp_sum32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// the lane's rotary pairs c = lane * PL + e of a row: elements c and c + D/2
template <int D>
struct Part {
  static constexpr int PL = D / 64;
  static constexpr int H = D / 2;
  float x0[PL], x1[PL];
  __device__ __forceinline__ void load(const __nv_bfloat16* row, int lane) {
#pragma unroll
    for (int e = 0; e < PL; ++e) {
      x0[e] = __bfloat162float(row[lane * PL + e]);
      x1[e] = __bfloat162float(row[lane * PL + e + H]);
    }
  }
  __device__ __forceinline__ Part rot(const float2* tab, int64_t pos, int lane, bool back = false) const {
    Part r;
#pragma unroll
    for (int e = 0; e < PL; ++e) {
      const float2 cs = tab ? tab[pos * H + lane * PL + e] : make_float2(1.f, 0.f);
      const float sn = back ? -cs.y : cs.y;
      r.x0[e] = x0[e] * cs.x - x1[e] * sn;
      r.x1[e] = x1[e] * cs.x + x0[e] * sn;
    }
    return r;
  }
  __device__ __forceinline__ float dot(const Part& o) const {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < PL; ++e) s = fmaf(x0[e], o.x0[e], fmaf(x1[e], o.x1[e], s));
    return s;
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int e = 0; e < PL; ++e) x0[e] = x1[e] = 0.f;
  }
  __device__ __forceinline__ void axpy(float a, const Part& o) {
#pragma unroll
    for (int e = 0; e < PL; ++e) {
      x0[e] = fmaf(a, o.x0[e], x0[e]);
      x1[e] = fmaf(a, o.x1[e], x1[e]);
    }
  }
  __device__ __forceinline__ void add(const Part& o) {
#pragma unroll
    for (int e = 0; e < PL; ++e) {
      x0[e] += o.x0[e];
      x1[e] += o.x1[e];
    }
  }
  __device__ __forceinline__ void store_bf16(__nv_bfloat16* row, int lane, float scale) const {
#pragma unroll
    for (int e = 0; e < PL; ++e) {
      row[lane * PL + e] = __float2bfloat16_rn(x0[e] * scale);
      row[lane * PL + e + H] = __float2bfloat16_rn(x1[e] * scale);
    }
  }
};

// retrieved keys of (b, h, s): cnt = blk * (valid blocks, which come first)
__device__ __forceinline__ int prefix_count(const SegBwdArgs& a, const int32_t* blocks) {
  const int nb = a.R / a.blk;
  int n = 0;
  for (int q = 0; q < nb; ++q) n += blocks[q] >= 0 ? 1 : 0;
  return n * a.blk;
}

template <int D>
__global__ void __launch_bounds__(256) seg_bwd_rows_kernel(SegBwdArgs a) {
  using PT = Part<D>;
  const int lane = threadIdx.x & 31;
  const int64_t nrows = (int64_t)a.B * a.Hq * a.T;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= nrows) return;  // whole warps only
  const int i = (int)(row % a.T);
  const int64_t bh = row / a.T;
  const int h = (int)(bh % a.Hq), b = (int)(bh / a.Hq);
  const int g = h / (a.Hq / a.Hkv);
  const int s = i / a.S;
  const int64_t sS = (int64_t)s * a.S;
  const bool is_long = a.long_slot[h] >= 0;
  PT q, go, o;
  q.load(a.Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st, lane);
  go.load(a.dO + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st, lane);
  o.load(a.O + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st, lane);
  const float dd = warp_sum32(go.dot(o));
  if (lane == 0) a.Dsum[row] = dd;
  const float nl2 = -a.lse[row] * kLog2e;
  const PT qi = q.rot(a.tab, i, lane);
  const __nv_bfloat16* Kg = a.K + b * a.k_sb + g * a.k_sh;
  const __nv_bfloat16* Vg = a.V + b * a.v_sb + g * a.v_sh;
  PT gq;
  gq.zero();
  auto pair = [&](int j, int64_t pos) {
    PT kr, vr;
    kr.load(Kg + (int64_t)j * a.k_st, lane);
    vr.load(Vg + (int64_t)j * a.v_st, lane);
    const PT ks = kr.rot(a.tab, pos, lane);
    const float z = warp_sum32(qi.dot(ks));
    const float p = exp2f(fmaf(z, a.scale_log2, nl2));
    const float dp = warp_sum32(go.dot(vr));
    gq.axpy(p * (dp - dd), ks);
  };
  int lo = (int)sS;
  if (is_long) {
    if (s > 0) {
      const int32_t* blocks = a.prefix_blocks + (bh * a.N + s) * (a.R / a.blk);
      const int cnt = prefix_count(a, blocks);
      for (int p = 0; p < cnt; ++p) pair(blocks[p / a.blk] * a.blk + p % a.blk, sS - cnt + p);
    }
  } else if (s > 0) {
    lo = (int)max((int64_t)0, sS - a.M);
  }
  for (int j = lo; j <= i; ++j) pair(j, j);
  const float scale = rsqrtf((float)a.d);
  gq.rot(a.tab, i, lane, true).store_bf16(a.dQ + b * a.dq_sb + h * a.dq_sh + (int64_t)i * a.dq_st, lane, scale);
}

template <int D>
__global__ void __launch_bounds__(256) seg_bwd_keys_kernel(SegBwdArgs a) {
  using PT = Part<D>;
  const int lane = threadIdx.x & 31;
  const int64_t nkeys = (int64_t)a.B * a.Hkv * a.T;
  const int64_t key = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (key >= nkeys) return;  // whole warps only
  const int j = (int)(key % a.T);
  const int64_t bg = key / a.T;
  const int g = (int)(bg % a.Hkv), b = (int)(bg / a.Hkv);
  const int rep = a.Hq / a.Hkv;
  const int sj = j / a.S;
  PT kr, vr;
  kr.load(a.K + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st, lane);
  vr.load(a.V + b * a.v_sb + g * a.v_sh + (int64_t)j * a.v_st, lane);
  const int nb = a.R / a.blk;
  PT gk, gv;  // gk in the raw frame
  gk.zero();
  gv.zero();
  for (int h = g * rep; h < (g + 1) * rep; ++h) {
    const int64_t bh = (int64_t)b * a.Hq + h;
    const bool is_long = a.long_slot[h] >= 0;
    // rows that keep j at its global position: its own segment from row j
    // on, and for local heads the later segments whose carried tail holds j
    const int s_hi = is_long ? sj : min(a.N - 1, (j + a.M) / a.S);
    const PT ks = kr.rot(a.tab, j, lane);
    PT acc;
    acc.zero();
    for (int s = sj; s <= s_hi; ++s) {
      const int i_lo = s == sj ? j : s * a.S;
      const int i_hi = (s + 1) * a.S;
      for (int i = i_lo; i < i_hi; ++i) {
        PT q, go;
        q.load(a.Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st, lane);
        go.load(a.dO + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st, lane);
        const PT qi = q.rot(a.tab, i, lane);
        const int64_t row = bh * a.T + i;
        const float z = warp_sum32(qi.dot(ks));
        const float p = exp2f(fmaf(z, a.scale_log2, -a.lse[row] * kLog2e));
        const float dp = warp_sum32(go.dot(vr));
        acc.axpy(p * (dp - a.Dsum[row]), qi);
        gv.axpy(p, go);
      }
    }
    gk.add(acc.rot(a.tab, j, lane, true));
    // rows whose segment retrieved j's block: the prefix slot gives the
    // rotary position j had there
    if (is_long && nb > 0) {
      const int blk_id = j / a.blk;
      for (int s = 1; s < a.N; ++s) {
        const int32_t* blocks = a.prefix_blocks + (bh * a.N + s) * nb;
        int slot_q = -1;
        for (int q = 0; q < nb; ++q)
          if (blocks[q] == blk_id) slot_q = q;
        if (slot_q < 0) continue;  // uniform over the warp
        const int cnt = prefix_count(a, blocks);
        const int64_t vpos = (int64_t)s * a.S - cnt + slot_q * a.blk + j % a.blk;
        const PT kv = kr.rot(a.tab, vpos, lane);
        PT accp;
        accp.zero();
        for (int i = s * a.S; i < (s + 1) * a.S; ++i) {
          PT q, go;
          q.load(a.Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st, lane);
          go.load(a.dO + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st, lane);
          const PT qi = q.rot(a.tab, i, lane);
          const int64_t row = bh * a.T + i;
          const float z = warp_sum32(qi.dot(kv));
          const float p = exp2f(fmaf(z, a.scale_log2, -a.lse[row] * kLog2e));
          const float dp = warp_sum32(go.dot(vr));
          accp.axpy(p * (dp - a.Dsum[row]), qi);
          gv.axpy(p, go);
        }
        gk.add(accp.rot(a.tab, vpos, lane, true));
      }
    }
  }
  const float scale = rsqrtf((float)a.d);
  gk.store_bf16(a.dK + b * a.dk_sb + g * a.dk_sh + (int64_t)j * a.dk_st, lane, scale);
  gv.store_bf16(a.dV + b * a.dv_sb + g * a.dv_sh + (int64_t)j * a.dv_st, lane, 1.f);
}

}  // namespace

cudaError_t launch_segment_bwd(const SegBwdArgs& a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.Hq * a.T;
  const int64_t keys = (int64_t)a.B * a.Hkv * a.T;
  if (rows == 0) return cudaSuccess;
  if (a.d == 128) {
    seg_bwd_rows_kernel<128><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(a);
    seg_bwd_keys_kernel<128><<<(unsigned)((keys + 7) / 8), 256, 0, st>>>(a);
  } else if (a.d == 64) {
    seg_bwd_rows_kernel<64><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(a);
    seg_bwd_keys_kernel<64><<<(unsigned)((keys + 7) / 8), 256, 0, st>>>(a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace sattn
