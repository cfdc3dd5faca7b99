// Fused Invariant Point Attention core for sm_100a.
//
// Three launches:
//   1. ipa_geometry_kernel  -- per batch: centroid of the valid frame origins,
//      query-tile (128 rows) and key-tile (64 rows) origins, per-residue
//      frames relative to the centroid, per-head point-term coefficient.
//   2. ipa_rows_kernel      -- one warp per (b, i, h): applies the frames and
//      writes the fp16 augmented rows Q_h, K_h, V_h (64 wide), the pair rows
//      Q_pair = w_L w_bias * z1 and Z2 = z2 (R*Cz wide), plus small fp32
//      per-row terms.
//   3. ipa_attention_kernel -- one CTA per (b, h, 128-query tile): a
//      flash-style pass over 64-key tiles with TMA-staged K/V, tcgen05 MMAs
//      accumulating in tensor memory, an online masked softmax on CUDA cores
//      and the fused epilogue.
//
// The squared point distance is folded into the augmented columns with the
// identity |a - b|^2 = |a|^2 + |b|^2 - 2 a.b (MEET, section 2.2 eq. (7)-(8)).
// To keep the fp32 accumulator of the tensor core small, point coordinates
// enter the MMA relative to the origin of their own tile (query tile o_I,
// key tile o_J); with d = o_J - o_I the exact logit is
//   MMA(2c gq'.gk' - c|gk'|^2) + c(2 sq.d - Pq|d|^2)   [per row and tile]
//                              - 2c sk.d               [per key and tile]
//   - c sum_p |gq'_p|^2                                 [per row: cancels]
// where c = log2(e) w_L gamma_h w_C / 2, sq = sum_p gq'_p, sk = sum_p gk'_p.
// The two small correction terms are added on CUDA cores in fp32.
#include <cuda_fp16.h>

#include <cmath>
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace fipa {

using namespace sm100;

namespace {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ldf(const View& v, int64_t off) {
  if (v.dtype == 1) return static_cast<float>(reinterpret_cast<const double*>(v.p)[off]);
  return reinterpret_cast<const float*>(v.p)[off];
}
__device__ __forceinline__ bool ldb(const View& v, int64_t off) {
  return reinterpret_cast<const unsigned char*>(v.p)[off] != 0;
}

// ------------------------------------------------------------- kernel 1
struct FrameArgs {
  int B, L, H, nqt, nkt;
  float w_L, w_C;
  View rot, trans, mask, gamma;
  float4* oq;     // [B, nqt]
  float4* ok;     // [B, nkt]
  float* frame;   // [B, L, 16]: R row-major (9), t - centroid (3), valid, 0, 0, 0
  float* headc;   // [H]
};

__global__ void __launch_bounds__(1024) ipa_geometry_kernel(const FrameArgs a) {
  const int b = blockIdx.x;
  const int tid = threadIdx.x, nth = blockDim.x;
  __shared__ double red[4][32];
  __shared__ float cen[3];

  double sx = 0, sy = 0, sz = 0, cnt = 0;
  for (int i = tid; i < a.L; i += nth) {
    if (!ldb(a.mask, b * a.mask.s[0] + i * a.mask.s[1])) continue;
    const int64_t o = b * a.trans.s[0] + i * a.trans.s[1];
    sx += ldf(a.trans, o);
    sy += ldf(a.trans, o + a.trans.s[2]);
    sz += ldf(a.trans, o + 2 * a.trans.s[2]);
    cnt += 1.0;
  }
  for (int off = 16; off > 0; off >>= 1) {
    sx += __shfl_xor_sync(0xffffffffu, sx, off);
    sy += __shfl_xor_sync(0xffffffffu, sy, off);
    sz += __shfl_xor_sync(0xffffffffu, sz, off);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
  }
  const int w = tid >> 5, lane = tid & 31;
  if (lane == 0) { red[0][w] = sx; red[1][w] = sy; red[2][w] = sz; red[3][w] = cnt; }
  __syncthreads();
  if (tid < 32) {
    const int nw = nth >> 5;
    double vx = lane < nw ? red[0][lane] : 0, vy = lane < nw ? red[1][lane] : 0;
    double vz = lane < nw ? red[2][lane] : 0, vc = lane < nw ? red[3][lane] : 0;
    for (int off = 16; off > 0; off >>= 1) {
      vx += __shfl_xor_sync(0xffffffffu, vx, off);
      vy += __shfl_xor_sync(0xffffffffu, vy, off);
      vz += __shfl_xor_sync(0xffffffffu, vz, off);
      vc += __shfl_xor_sync(0xffffffffu, vc, off);
    }
    if (lane == 0) {
      const double inv = vc > 0 ? 1.0 / vc : 0.0;
      cen[0] = static_cast<float>(vx * inv);
      cen[1] = static_cast<float>(vy * inv);
      cen[2] = static_cast<float>(vz * inv);
    }
  }
  __syncthreads();
  const float cx = cen[0], cy = cen[1], cz = cen[2];

  // per-residue frames relative to the centroid
  for (int i = tid; i < a.L; i += nth) {
    float* f = a.frame + (static_cast<int64_t>(b) * a.L + i) * 16;
    const int64_t ro = b * a.rot.s[0] + i * a.rot.s[1];
    for (int x = 0; x < 3; ++x)
      for (int y = 0; y < 3; ++y) f[x * 3 + y] = ldf(a.rot, ro + x * a.rot.s[2] + y * a.rot.s[3]);
    const int64_t o = b * a.trans.s[0] + i * a.trans.s[1];
    f[9] = ldf(a.trans, o) - cx;
    f[10] = ldf(a.trans, o + a.trans.s[2]) - cy;
    f[11] = ldf(a.trans, o + 2 * a.trans.s[2]) - cz;
    f[12] = ldb(a.mask, b * a.mask.s[0] + i * a.mask.s[1]) ? 1.f : 0.f;
    f[13] = f[14] = f[15] = 0.f;
  }

  // tile origins: mean of the centred origins of the valid residues in the tile
  const int nw = nth >> 5;
  for (int t = w; t < a.nqt + a.nkt; t += nw) {
    const bool isq = t < a.nqt;
    const int T = isq ? QT : KT;
    const int tile = isq ? t : t - a.nqt;
    float ax = 0, ay = 0, az = 0, an = 0;
    for (int r = lane; r < T; r += 32) {
      const int i = tile * T + r;
      if (i >= a.L) break;
      if (!ldb(a.mask, b * a.mask.s[0] + i * a.mask.s[1])) continue;
      const int64_t o = b * a.trans.s[0] + i * a.trans.s[1];
      ax += ldf(a.trans, o) - cx;
      ay += ldf(a.trans, o + a.trans.s[2]) - cy;
      az += ldf(a.trans, o + 2 * a.trans.s[2]) - cz;
      an += 1.f;
    }
    for (int off = 16; off > 0; off >>= 1) {
      ax += __shfl_xor_sync(0xffffffffu, ax, off);
      ay += __shfl_xor_sync(0xffffffffu, ay, off);
      az += __shfl_xor_sync(0xffffffffu, az, off);
      an += __shfl_xor_sync(0xffffffffu, an, off);
    }
    if (lane == 0) {
      const float inv = an > 0 ? 1.f / an : 0.f;
      const float4 o4 = make_float4(ax * inv, ay * inv, az * inv, 0.f);
      if (isq) a.oq[b * a.nqt + tile] = o4;
      else a.ok[b * a.nkt + tile] = o4;
    }
  }

  if (b == 0) {
    for (int h = tid; h < a.H; h += nth)
      a.headc[h] = kLog2e * a.w_L * ldf(a.gamma, h * a.gamma.s[0]) * a.w_C * 0.5f;
  }
}

// ------------------------------------------------------------- kernel 2
struct RowArgs {
  int B, L, H, C, Pq, Pv, R, Cz, RCz, DZ, nqt, nkt;
  float qscale;     // log2(e) w_L scalar_scale
  float bscale;     // log2(e) w_L
  View q, k, v, q_pts, k_pts, v_pts, z1, z2, w_bias;
  const float* frame;
  const float4* oq;
  const float4* ok;
  const float* headc;
  __half* qh;       // [B*H, L, 64]
  __half* kh;
  __half* vh;
  __half* qp;       // [B*H, L, DZ]
  __half* z2o;      // [B, L, DZ]
  float* z1f;       // [B, L, RCz]
  float4* rowq;     // [B*H, L]
  float4* colk;     // [B*H, L]
  int* err;
};

struct Split {
  __half hi, lo;
};
__device__ __forceinline__ Split split_f16(float x) {
  Split s;
  s.hi = __float2half_rn(x);
  s.lo = __float2half_rn(x - __half2float(s.hi));
  return s;
}

__global__ void __launch_bounds__(128) ipa_rows_kernel(const RowArgs a) {
  const int warp_global = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t total = static_cast<int64_t>(a.B) * a.L * a.H;
  if (warp_global >= total) return;
  const int h = warp_global % a.H;
  const int i = (warp_global / a.H) % a.L;
  const int b = warp_global / (a.H * a.L);
  const int64_t bh = static_cast<int64_t>(b) * a.H + h;
  const int64_t rowi = bh * a.L + i;

  const float* f = a.frame + (static_cast<int64_t>(b) * a.L + i) * 16;
  float Rm[9];
#pragma unroll
  for (int e = 0; e < 9; ++e) Rm[e] = f[e];
  const float tx = f[9], ty = f[10], tz = f[11];
  const bool valid = f[12] != 0.f;
  const float4 oqv = a.oq[b * a.nqt + i / QT];
  const float4 okv = a.ok[b * a.nkt + i / KT];
  const float c = a.headc[h];

  const int C = a.C, Pq = a.Pq, Pv = a.Pv;
  const int64_t qb = b * a.q.s[0] + i * a.q.s[1] + h * a.q.s[2];
  const int64_t kb = b * a.k.s[0] + i * a.k.s[1] + h * a.k.s[2];
  const int64_t vb = b * a.v.s[0] + i * a.v.s[1] + h * a.v.s[2];
  const int64_t qpb = b * a.q_pts.s[0] + i * a.q_pts.s[1] + h * a.q_pts.s[2];
  const int64_t kpb = b * a.k_pts.s[0] + i * a.k_pts.s[1] + h * a.k_pts.s[2];
  const int64_t vpb = b * a.v_pts.s[0] + i * a.v_pts.s[1] + h * a.v_pts.s[2];
  const float tt[3] = {tx, ty, tz};
  const float oqa[3] = {oqv.x, oqv.y, oqv.z};
  const float oka[3] = {okv.x, okv.y, okv.z};

  // global point coordinate x of point p: sum_y R[x][y] pts[p][y] + t'[x] - origin[x]
  auto gpt = [&](const View& P, int64_t base, int p, int x, float origin) -> float {
    const int64_t o = base + p * P.s[3];
    const float p0 = ldf(P, o), p1 = ldf(P, o + P.s[4]), p2 = ldf(P, o + 2 * P.s[4]);
    return fmaf(Rm[x * 3 + 0], p0, fmaf(Rm[x * 3 + 1], p1, Rm[x * 3 + 2] * p2)) + tt[x] - origin;
  };

  bool overflow = false;
  // ---- Q_h, K_h, V_h: lane writes columns 2*lane, 2*lane+1
  {
    float qv[2], kv[2], vv[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int col = 2 * lane + e;
      float qx = 0.f, kx = 0.f, vx = 0.f;
      if (valid) {
        // query row: [ scalar | gq' hi | gq' hi | gq' lo | -1 -1 | 0 ]
        if (col < C) {
          qx = a.qscale * ldf(a.q, qb + col * a.q.s[3]);
        } else if (col < C + 9 * Pq) {
          const int u = col - C, part = u / (3 * Pq), e3 = u % (3 * Pq);
          const Split sp = split_f16(gpt(a.q_pts, qpb, e3 / 3, e3 % 3, oqa[e3 % 3]));
          qx = __half2float(part < 2 ? sp.hi : sp.lo);
        } else if (col < C + 9 * Pq + 2) {
          qx = -1.f;
        }
        // key row: [ scalar | 2c gk' hi | lo | hi | c|gk'|^2 hi, lo | 0 ]
        if (col < C) {
          kx = ldf(a.k, kb + col * a.k.s[3]);
        } else if (col < C + 9 * Pq) {
          const int u = col - C, part = u / (3 * Pq), e3 = u % (3 * Pq);
          const Split sp = split_f16(2.f * c * gpt(a.k_pts, kpb, e3 / 3, e3 % 3, oka[e3 % 3]));
          kx = __half2float(part == 1 ? sp.lo : sp.hi);
        } else if (col < C + 9 * Pq + 2) {
          float n = 0.f;
          for (int p = 0; p < Pq; ++p)
            for (int x = 0; x < 3; ++x) {
              const float g = gpt(a.k_pts, kpb, p, x, oka[x]);
              n = fmaf(g, g, n);
            }
          const Split sp = split_f16(c * n);
          kx = __half2float(col == C + 9 * Pq ? sp.hi : sp.lo);
        }
        // value row: [ scalar | gv hi | gv lo | 0 ], gv relative to the centroid
        if (col < C) {
          vx = ldf(a.v, vb + col * a.v.s[3]);
        } else if (col < C + 6 * Pv) {
          const int u = col - C, part = u / (3 * Pv), e3 = u % (3 * Pv);
          const Split sp = split_f16(gpt(a.v_pts, vpb, e3 / 3, e3 % 3, 0.f));
          vx = __half2float(part == 0 ? sp.hi : sp.lo);
        }
      }
      qv[e] = qx;
      kv[e] = kx;
      vv[e] = vx;
    }
    const __half2 q2 = __floats2half2_rn(qv[0], qv[1]);
    const __half2 k2 = __floats2half2_rn(kv[0], kv[1]);
    const __half2 v2 = __floats2half2_rn(vv[0], vv[1]);
    overflow |= __hisinf(q2.x) || __hisinf(q2.y) || __hisinf(k2.x) || __hisinf(k2.y) ||
                __hisinf(v2.x) || __hisinf(v2.y);
    reinterpret_cast<__half2*>(a.qh + rowi * DH)[lane] = q2;
    reinterpret_cast<__half2*>(a.kh + rowi * DH)[lane] = k2;
    reinterpret_cast<__half2*>(a.vh + rowi * DH)[lane] = v2;
  }

  // ---- Q_pair (this head), and Z2 / z1 copies (head 0 only)
  for (int c0 = lane * 8; c0 < a.DZ; c0 += 256) {
    uint32_t w4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float vals[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int u = c0 + 2 * e + t;
        float val = 0.f;
        if (valid && u < a.RCz) {
          const int r = u / a.Cz, cc = u % a.Cz;
          val = a.bscale * ldf(a.w_bias, cc * a.w_bias.s[0] + h * a.w_bias.s[1]) *
                ldf(a.z1, b * a.z1.s[0] + i * a.z1.s[1] + r * a.z1.s[2] + cc * a.z1.s[3]);
        }
        vals[t] = val;
      }
      w4[e] = pack_half2(vals[0], vals[1]);
    }
    *reinterpret_cast<uint4*>(a.qp + rowi * a.DZ + c0) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
  if (h == 0) {
    const int64_t zr = static_cast<int64_t>(b) * a.L + i;
    for (int c0 = lane * 8; c0 < a.DZ; c0 += 256) {
      uint32_t w4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float vals[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int u = c0 + 2 * e + t;
          float val = 0.f;
          if (valid && u < a.RCz) {
            const int r = u / a.Cz, cc = u % a.Cz;
            val = ldf(a.z2, b * a.z2.s[0] + i * a.z2.s[1] + r * a.z2.s[2] + cc * a.z2.s[3]);
          }
          vals[t] = val;
        }
        w4[e] = pack_half2(vals[0], vals[1]);
      }
      *reinterpret_cast<uint4*>(a.z2o + zr * a.DZ + c0) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    for (int u = lane; u < a.RCz; u += 32) {
      const int r = u / a.Cz, cc = u % a.Cz;
      a.z1f[zr * a.RCz + u] =
          valid ? ldf(a.z1, b * a.z1.s[0] + i * a.z1.s[1] + r * a.z1.s[2] + cc * a.z1.s[3]) : 0.f;
    }
  }

  // ---- per-row terms: sq = sum_p gq'_p ; sk_hat = 2c sum_p gk'_p, key mask bias
  if (lane < 2) {
    float s[3] = {0.f, 0.f, 0.f};
    if (valid) {
      for (int p = 0; p < Pq; ++p)
        for (int x = 0; x < 3; ++x)
          s[x] += lane == 0 ? gpt(a.q_pts, qpb, p, x, oqa[x]) : gpt(a.k_pts, kpb, p, x, oka[x]);
    }
    if (lane == 0) {
      a.rowq[rowi] = make_float4(s[0], s[1], s[2], 0.f);
    } else {
      a.colk[rowi] = make_float4(2.f * c * s[0], 2.f * c * s[1], 2.f * c * s[2],
                                 valid ? 0.f : -INFINITY);
    }
  }
  if (__any_sync(0xffffffffu, overflow) && lane == 0) record_error(a.err, DEV_NONFINITE);
}

// ------------------------------------------------------------- kernel 3
struct AttnArgs {
  int B, L, H, DZ, RCz, Cz, nqt, nkt, F;
  float tau;
  const float4* rowq;
  const float4* colk;
  const float4* oq;
  const float4* ok;
  const float* headc;
  const __half* qp;
  const float* frame;
  const float* z1f;
  float* out;
  int* err;
};

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t SM_QH = 0;                          // 128 x 64 fp16, SW128
constexpr uint32_t STG_BYTES = 16384 + 8192 * 4;       // Kh | Vh | Z2 (<= 4 panels)
constexpr uint32_t SM_STG = 16384;
constexpr uint32_t SM_P = SM_STG + NSTAGE * STG_BYTES; // 2 x (128 x 64 fp16, SW128)
constexpr uint32_t SM_AUX = SM_P + 2 * 16384;
constexpr uint32_t AUX_COL = 0;                        // float [NSTAGE][64]
constexpr uint32_t AUX_D = 1024;                       // float4 [NSTAGE]
constexpr uint32_t AUX_BAR = 1152;                     // mbarriers
constexpr uint32_t SMEM_BYTES = SM_AUX + 2048;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;     // + alignment slack

// barrier slots
enum { B_Q = 0, B_QP, B_SFULL, B_SFREE, B_FULL0, B_EMPTY0 = B_FULL0 + NSTAGE,
       B_PFULL0 = B_EMPTY0 + NSTAGE, B_PFREE0 = B_PFULL0 + 2, B_DRAIN = B_PFREE0 + 2,
       B_COUNT = B_DRAIN + 1 };
constexpr uint32_t AUX_TMEM = AUX_BAR + 8 * B_COUNT;
constexpr uint32_t AUX_ABORT = AUX_TMEM + 8;

// tensor memory columns
constexpr uint32_t TM_O = 0;      // O: [Vh part 64 | pair part DZ]
constexpr uint32_t TM_S = 320;    // S: 64 fp32 columns
constexpr uint32_t TM_QP = 384;   // Q_pair: DZ/2 packed-fp16 columns
constexpr uint32_t TM_COLS = 512;

__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) {  // K-major SW128
  return smem_desc_sw128(saddr, 16, 1024);
}
__device__ __forceinline__ uint64_t mndesc(uint32_t saddr) {  // MN-major SW128, 64-col panels 8 KB apart
  return smem_desc_sw128(saddr, 8192, 1024);
}

__global__ void __launch_bounds__(192, 1)
    ipa_attention_kernel(const __grid_constant__ CUtensorMap tm_qh,
                         const __grid_constant__ CUtensorMap tm_kh,
                         const __grid_constant__ CUtensorMap tm_vh,
                         const __grid_constant__ CUtensorMap tm_z2, const AttnArgs a) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sb = (raw_u32 + 1023u) & ~1023u;             // shared address of the base
  unsigned char* smem = smem_raw + (sb - raw_u32);             // generic pointer of the base

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int I = blockIdx.x % a.nqt;
  const int bh = blockIdx.x / a.nqt;
  const int b = bh / a.H, h = bh % a.H;
  const int L = a.L, nt = a.nkt, DZ = a.DZ;

  float* col_s = reinterpret_cast<float*>(smem + SM_AUX + AUX_COL);
  float4* dinfo = reinterpret_cast<float4*>(smem + SM_AUX + AUX_D);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM_AUX + AUX_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM_AUX + AUX_TMEM);
  auto bar = [&](int k) -> uint32_t { return sb + SM_AUX + AUX_BAR + 8u * k; };

  if (tid == 0) {
    mbar_init(bar(B_Q), 1);
    mbar_init(bar(B_QP), 128);
    mbar_init(bar(B_SFULL), 1);
    mbar_init(bar(B_SFREE), 128);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(bar(B_FULL0 + s), 1);
      mbar_init(bar(B_EMPTY0 + s), 1);
    }
    for (int p = 0; p < 2; ++p) {
      mbar_init(bar(B_PFULL0 + p), 128);
      mbar_init(bar(B_PFREE0 + p), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), TM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_qh);
    tma_prefetch_desc(&tm_kh);
    tma_prefetch_desc(&tm_vh);
    tma_prefetch_desc(&tm_z2);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&](int code) {
    record_error(a.err, code);
    *abort_flag = 1;
  };

  if (warp == 4) {
    // ------------------------------------------------ TMA producer warp
    const float4 oqv = a.oq[b * a.nqt + I];
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(B_Q), 16384);
      tma_load_3d(sb + SM_QH, &tm_qh, bar(B_Q), 0, I * QT, bh);
    }
    int issued = 0;
    for (int j = 0; j < nt; ++j) {
      const int s = j % NSTAGE;
      const int J = (2 * I + j) % nt;
      if (j >= NSTAGE) {
        int ok = 1;
        if (lane == 0) ok = mbar_wait_bounded(bar(B_EMPTY0 + s), ((j / NSTAGE) - 1) & 1, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) fail(DEV_TIMEOUT_EMPTY);
          break;
        }
      }
      const float4 okv = a.ok[b * nt + J];
      const float dx = okv.x - oqv.x, dy = okv.y - oqv.y, dz = okv.z - oqv.z;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int kk = lane + 32 * t;
        const int key = J * KT + kk;
        float cv = -INFINITY;
        if (key < L) {
          const float4 ck = a.colk[static_cast<int64_t>(bh) * L + key];
          cv = ck.w - fmaf(ck.x, dx, fmaf(ck.y, dy, ck.z * dz));
        }
        col_s[s * KT + kk] = cv;
      }
      if (lane == 0) dinfo[s] = make_float4(dx, dy, dz, fmaf(dx, dx, fmaf(dy, dy, dz * dz)));
      __syncwarp();
      if (lane == 0) {
        const uint32_t st = sb + SM_STG + s * STG_BYTES;
        mbar_arrive_expect_tx(bar(B_FULL0 + s), 16384u + static_cast<uint32_t>(DZ) * 128u);
        tma_load_3d(st, &tm_kh, bar(B_FULL0 + s), 0, J * KT, bh);
        tma_load_3d(st + 8192, &tm_vh, bar(B_FULL0 + s), 0, J * KT, bh);
        for (int p = 0; p < DZ / 64; ++p)
          tma_load_3d(st + 16384 + 8192 * p, &tm_z2, bar(B_FULL0 + s), 64 * p, J * KT, b);
      }
      __syncwarp();
      issued = j + 1;
    }
    // drain: make sure no TMA write is still in flight when the CTA leaves
    if (lane == 0 && *abort_flag) {
      for (int j = (issued > NSTAGE ? issued - NSTAGE : 0); j < issued; ++j)
        mbar_wait_bounded(bar(B_FULL0 + j % NSTAGE), (j / NSTAGE) & 1, nullptr, 100000000ull);
    }
  } else if (warp == 5) {
    // ------------------------------------------------ MMA issuer (one thread)
    if (lane == 0) {
      bool ok = mbar_wait_bounded(bar(B_Q), 0, abort_flag) && mbar_wait_bounded(bar(B_QP), 0, abort_flag);
      if (!ok) fail(DEV_TIMEOUT_SOFTMAX);
      tc_fence_after();
      const uint32_t idq = idesc_f16(128, KT, false);
      const uint32_t idv1 = idesc_f16(128, 64, true);
      const uint32_t idv2 = idesc_f16(128, DZ, true);
      const uint32_t tS = tmem + TM_S, tO = tmem + TM_O, tQP = tmem + TM_QP;
      bool issued_any = false;
      for (int j = 0; ok && j <= nt; ++j) {
        if (j < nt) {
          const int s = j % NSTAGE;
          ok = mbar_wait_bounded(bar(B_FULL0 + s), (j / NSTAGE) & 1, abort_flag);
          if (ok && j > 0) ok = mbar_wait_bounded(bar(B_SFREE), (j - 1) & 1, abort_flag);
          if (!ok) { fail(DEV_TIMEOUT_FULL); break; }
          tc_fence_after();
          const uint32_t st = sb + SM_STG + s * STG_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_ss(tS, kdesc(sb + SM_QH + 32 * k), kdesc(st + 32 * k), idq, k > 0 ? 1u : 0u);
          for (int kk = 0; kk < DZ / 16; ++kk)
            umma_ts(tS, tQP + 8 * kk, kdesc(st + 16384 + 8192 * (kk >> 2) + 32 * (kk & 3)), idq, 1u);
          umma_commit(bar(B_SFULL));
          issued_any = true;
        }
        if (j > 0) {
          const int jj = j - 1, pb = jj & 1, s2 = jj % NSTAGE;
          ok = mbar_wait_bounded(bar(B_PFULL0 + pb), (jj >> 1) & 1, abort_flag);
          if (!ok) { fail(DEV_TIMEOUT_SOFTMAX); break; }
          tc_fence_after();
          const uint32_t pbase = sb + SM_P + 16384 * pb;
          const uint32_t st = sb + SM_STG + s2 * STG_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t acc = (jj > 0 || k > 0) ? 1u : 0u;
            umma_ss(tO, kdesc(pbase + 32 * k), mndesc(st + 8192 + 2048 * k), idv1, acc);
            umma_ss(tO + 64, kdesc(pbase + 32 * k), mndesc(st + 16384 + 2048 * k), idv2, acc);
          }
          umma_commit(bar(B_PFREE0 + pb));
          umma_commit(bar(B_EMPTY0 + s2));
        }
      }
      if (!ok && issued_any) {
        // wait (bounded) until every MMA already issued has retired
        umma_commit(bar(B_DRAIN));
        mbar_wait_bounded(bar(B_DRAIN), 0, nullptr, 100000000ull);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax + epilogue (128 threads)
    const int row = I * QT + tid;
    const bool in_range = row < L;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float ch = a.headc[h];
    const float4 sq = in_range ? a.rowq[static_cast<int64_t>(bh) * L + row] : make_float4(0, 0, 0, 0);
    const float pq = static_cast<float>(IPA_PQ);

    // Q_pair row -> tensor memory (A operand of the pair part of Q K^T)
    {
      const uint4* src = reinterpret_cast<const uint4*>(a.qp + (static_cast<int64_t>(bh) * L + row) * DZ);
      for (int c0 = 0; c0 < DZ / 2; c0 += 32) {
        uint32_t r[32];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint4 v = in_range ? src[c0 / 4 + e] : make_uint4(0, 0, 0, 0);
          r[4 * e + 0] = v.x;
          r[4 * e + 1] = v.y;
          r[4 * e + 2] = v.z;
          r[4 * e + 3] = v.w;
        }
        tmem_st32(tmem + TM_QP + c0 + lane_off, r);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_QP));
    }

    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    const int OW = 64 + DZ;
    for (int j = 0; j < nt && ok; ++j) {
      const int s = j % NSTAGE, pb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(B_SFULL), j & 1, abort_flag))) {
        if (lane == 0) fail(DEV_TIMEOUT_MMA);
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[64];
      {
        uint32_t r0[32], r1[32];
        tmem_ld32(tmem + TM_S + lane_off, r0);
        tmem_ld32(tmem + TM_S + 32 + lane_off, r1);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) { sr[e] = r0[e]; sr[32 + e] = r1[e]; }
      }
      tc_fence_before();
      mbar_arrive(bar(B_SFREE));
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(B_FULL0 + s), (j / NSTAGE) & 1, abort_flag))) {
        if (lane == 0) fail(DEV_TIMEOUT_FULL);
        ok = false;
        break;
      }

      const float* colv = col_s + s * KT;
      const float4 dd = dinfo[s];
      const float r = ch * (2.f * fmaf(sq.x, dd.x, fmaf(sq.y, dd.y, sq.z * dd.z)) - pq * dd.w);
      float x[64];
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < 64; ++k) {
        x[k] = __uint_as_float(sr[k]) + colv[k];
        mx = fmaxf(mx, x[k]);
      }
      const float mt = mx + r;
      const bool need = mt > m_used + a.tau;
      const bool resc = need && (m_used != -INFINITY);
      const float scale = resc ? ex2(m_used - mt) : 1.f;
      if (need) m_used = mt;
      l *= scale;
      if (__any_sync(0xffffffffu, resc)) {
        // O must be complete up to tile j-1 before it is rescaled
        if (!__all_sync(0xffffffffu,
                        mbar_wait_bounded(bar(B_PFREE0 + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag))) {
          if (lane == 0) fail(DEV_TIMEOUT_MMA);
          ok = false;
          break;
        }
        tc_fence_after();
        for (int c0 = 0; c0 < OW; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + TM_O + c0 + lane_off, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * scale);
          tmem_st32(tmem + TM_O + c0 + lane_off, o);
        }
        tmem_st_wait();
        tc_fence_before();
      }
      const float base = m_used - r;
      const bool live = m_used != -INFINITY;
      uint32_t pk[32];
      float ls = 0.f;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float p0 = live ? ex2(x[2 * k] - base) : 0.f;
        const float p1 = live ? ex2(x[2 * k + 1] - base) : 0.f;
        pk[k] = pack_half2(p0, p1);
        const float2 fr = unpack_half2(pk[k]);
        ls += fr.x + fr.y;
      }
      l += ls;
      if (j >= 2) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(B_PFREE0 + pb), ((j - 2) >> 1) & 1, abort_flag))) {
          if (lane == 0) fail(DEV_TIMEOUT_MMA);
          ok = false;
          break;
        }
      }
      unsigned char* prow = smem + SM_P + 16384 * pb + tid * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(prow + ((c ^ (tid & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_proxy_async_smem();
      mbar_arrive(bar(B_PFULL0 + pb));
    }

    // ------------------------------------------------ epilogue
    if (ok && !__all_sync(0xffffffffu, mbar_wait_bounded(bar(B_PFREE0 + ((nt - 1) & 1)),
                                                          ((nt - 1) >> 1) & 1, abort_flag))) {
      if (lane == 0) fail(DEV_TIMEOUT_MMA);
      ok = false;
    }
    const bool all_ok = __all_sync(0xffffffffu, ok);
    const float* fr = a.frame + (static_cast<int64_t>(b) * L + (in_range ? row : 0)) * 16;
    const bool dead = !(in_range && fr[12] != 0.f && l > 0.f);
    const int pitch = OW + 4;
    float* stage = reinterpret_cast<float*>(smem + SM_STG);
    if (all_ok) {
      tc_fence_after();
      const float inv = dead ? 0.f : 1.f / l;
      float* orow = stage + tid * pitch;
      for (int c0 = 0; c0 < OW; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + TM_O + c0 + lane_off, o);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(orow + c0 + e) =
              make_float4(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv,
                          __uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
      }
      orow[OW] = dead ? 1.f : 0.f;
    }
    tc_fence_before();
    named_bar_sync(1, 128);
    if (!*abort_flag) {
      const int C = IPA_C, Pv = IPA_PV, Cz = a.Cz;
      const int F = a.F;
      for (int rr = 0; rr < 32; ++rr) {
        const int rloc = warp * 32 + rr;
        const int grow = I * QT + rloc;
        if (grow >= L) break;
        const float* O = stage + rloc * pitch;
        const bool rdead = O[OW] != 0.f;
        const float* fg = a.frame + (static_cast<int64_t>(b) * L + grow) * 16;
        float* dst = a.out + ((static_cast<int64_t>(b) * L + grow) * a.H + h) * F;
        const float* z1r = a.z1f + (static_cast<int64_t>(b) * L + grow) * a.RCz;
        for (int f = lane; f < F; f += 32) {
          float val = 0.f;
          if (!rdead) {
            if (f < C) {
              val = O[f];
            } else if (f < C + 4 * Pv) {
              const bool is_norm = f >= C + 3 * Pv;
              const int p = is_norm ? f - C - 3 * Pv : (f - C) / 3;
              float op[3];
#pragma unroll
              for (int xx = 0; xx < 3; ++xx) {
                float acc = 0.f;
#pragma unroll
                for (int y = 0; y < 3; ++y) {
                  const float og = O[C + 3 * p + y] + O[C + 3 * Pv + 3 * p + y];
                  acc = fmaf(fg[y * 3 + xx], og - fg[9 + y], acc);
                }
                op[xx] = acc;
              }
              val = is_norm ? sqrtf(fmaf(op[0], op[0], fmaf(op[1], op[1], op[2] * op[2])))
                            : op[(f - C) % 3];
            } else {
              const int cc = f - C - 4 * Pv;
              for (int rr2 = 0; rr2 < a.RCz / Cz; ++rr2)
                val = fmaf(z1r[rr2 * Cz + cc], O[64 + rr2 * Cz + cc], val);
            }
          }
          dst[f] = val;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace

IpaWorkspace ipa_workspace_layout(int B, int L, int H, int DZ, int RCz) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  IpaWorkspace w{};
  size_t o = 0;
  const size_t bhl = static_cast<size_t>(B) * H * L, bl = static_cast<size_t>(B) * L;
  const int nqt = (L + QT - 1) / QT, nkt = (L + KT - 1) / KT;
  w.qh = o; o = up(o + bhl * DH * 2);
  w.kh = o; o = up(o + bhl * DH * 2);
  w.vh = o; o = up(o + bhl * DH * 2);
  w.qp = o; o = up(o + bhl * DZ * 2);
  w.z2 = o; o = up(o + bl * DZ * 2);
  w.rowq = o; o = up(o + bhl * 16);
  w.colk = o; o = up(o + bhl * 16);
  w.frame = o; o = up(o + bl * 64);
  w.z1f = o; o = up(o + bl * RCz * 4);
  w.oq = o; o = up(o + static_cast<size_t>(B) * nqt * 16);
  w.ok = o; o = up(o + static_cast<size_t>(B) * nkt * 16);
  w.headc = o; o = up(o + static_cast<size_t>(H) * 4);
  w.err = o; o = up(o + 16);
  w.total = o;
  return w;
}

cudaError_t ipa_launch_prologue(const IpaLaunch& a, cudaStream_t stream) {
  unsigned char* ws = a.ws;
  const IpaWorkspace& w = a.lay;

  FrameArgs g{};
  g.B = a.B; g.L = a.L; g.H = a.H; g.nqt = a.nqt; g.nkt = a.nkt;
  g.w_L = a.w_L; g.w_C = a.w_C;
  g.rot = a.rot; g.trans = a.trans; g.mask = a.mask; g.gamma = a.gamma;
  g.oq = reinterpret_cast<float4*>(ws + w.oq);
  g.ok = reinterpret_cast<float4*>(ws + w.ok);
  g.frame = reinterpret_cast<float*>(ws + w.frame);
  g.headc = reinterpret_cast<float*>(ws + w.headc);
  ipa_geometry_kernel<<<a.B, 1024, 0, stream>>>(g);

  RowArgs r{};
  r.B = a.B; r.L = a.L; r.H = a.H; r.C = a.C; r.Pq = a.Pq; r.Pv = a.Pv; r.R = a.R; r.Cz = a.Cz;
  r.RCz = a.RCz; r.DZ = a.DZ; r.nqt = a.nqt; r.nkt = a.nkt;
  r.qscale = kLog2e * a.w_L * a.scalar_scale;
  r.bscale = kLog2e * a.w_L;
  r.q = a.q; r.k = a.k; r.v = a.v; r.q_pts = a.q_pts; r.k_pts = a.k_pts; r.v_pts = a.v_pts;
  r.z1 = a.z1; r.z2 = a.z2; r.w_bias = a.w_bias;
  r.frame = g.frame; r.oq = g.oq; r.ok = g.ok; r.headc = g.headc;
  r.qh = reinterpret_cast<__half*>(ws + w.qh);
  r.kh = reinterpret_cast<__half*>(ws + w.kh);
  r.vh = reinterpret_cast<__half*>(ws + w.vh);
  r.qp = reinterpret_cast<__half*>(ws + w.qp);
  r.z2o = reinterpret_cast<__half*>(ws + w.z2);
  r.z1f = reinterpret_cast<float*>(ws + w.z1f);
  r.rowq = reinterpret_cast<float4*>(ws + w.rowq);
  r.colk = reinterpret_cast<float4*>(ws + w.colk);
  r.err = a.err;
  const int64_t warps = static_cast<int64_t>(a.B) * a.L * a.H;
  ipa_rows_kernel<<<static_cast<unsigned>((warps + 3) / 4), 128, 0, stream>>>(r);
  return cudaGetLastError();
}

cudaError_t ipa_launch_core(const IpaLaunch& a, cudaStream_t stream) {
  unsigned char* ws = a.ws;
  const IpaWorkspace& w = a.lay;
  __half* qh = reinterpret_cast<__half*>(ws + w.qh);
  __half* kh = reinterpret_cast<__half*>(ws + w.kh);
  __half* vh = reinterpret_cast<__half*>(ws + w.vh);
  __half* z2o = reinterpret_cast<__half*>(ws + w.z2);
  CUtensorMap tqh, tkh, tvh, tz2;
  const uint64_t bh = static_cast<uint64_t>(a.B) * a.H;
  bool ok = encode_tmap_f16_3d(&tqh, qh, DH, a.L, bh, DH * 2, static_cast<uint64_t>(a.L) * DH * 2, 64, QT) &&
            encode_tmap_f16_3d(&tkh, kh, DH, a.L, bh, DH * 2, static_cast<uint64_t>(a.L) * DH * 2, 64, KT) &&
            encode_tmap_f16_3d(&tvh, vh, DH, a.L, bh, DH * 2, static_cast<uint64_t>(a.L) * DH * 2, 64, KT) &&
            encode_tmap_f16_3d(&tz2, z2o, a.DZ, a.L, a.B, static_cast<uint64_t>(a.DZ) * 2,
                               static_cast<uint64_t>(a.L) * a.DZ * 2, 64, KT);
  if (!ok) return cudaErrorInvalidValue;

  {
    cudaError_t e = cudaFuncSetAttribute(ipa_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(SMEM_ALLOC));
    if (e != cudaSuccess) return e;
  }
  AttnArgs t{};
  t.B = a.B; t.L = a.L; t.H = a.H; t.DZ = a.DZ; t.RCz = a.RCz; t.Cz = a.Cz;
  t.nqt = a.nqt; t.nkt = a.nkt; t.F = a.F; t.tau = 8.f;
  t.rowq = reinterpret_cast<const float4*>(ws + w.rowq);
  t.colk = reinterpret_cast<const float4*>(ws + w.colk);
  t.oq = reinterpret_cast<const float4*>(ws + w.oq);
  t.ok = reinterpret_cast<const float4*>(ws + w.ok);
  t.headc = reinterpret_cast<const float*>(ws + w.headc);
  t.qp = reinterpret_cast<const __half*>(ws + w.qp);
  t.frame = reinterpret_cast<const float*>(ws + w.frame);
  t.z1f = reinterpret_cast<const float*>(ws + w.z1f);
  t.out = a.out; t.err = a.err;
  ipa_attention_kernel<<<static_cast<unsigned>(bh * a.nqt), 192, SMEM_ALLOC, stream>>>(tqh, tkh, tvh, tz2, t);
  return cudaGetLastError();
}

}  // namespace fipa
