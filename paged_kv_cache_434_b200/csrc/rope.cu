// rope.cu -- rotary position embedding fused with the cache write.
//
// "AI Infra入门干货总结：大模型是如何高效推理的", section "Reshape & Cache": the
// fused QKV output is split by columns, Q and K are rotated by the rotation of
// the token's position (element-wise sin/cos, dimensions unchanged), V is
// not, and reshape_and_cache scatters K and V into the paged pools through
// slot_mapping.  The sin/cos come from a cos_sin_cache [max_position,
// rotary_dim] built once (so that no sin/cos runs per token); the ursb.me
// Field Note blurb describes each Q/K pair as a complex number turned by
// position * theta_i.
//
// One pass over the step's tokens, CTAs walking tokens: each Q/K/V row is read
// once; rotated K and plain V go straight to the token's slot in the pools
// and the rotated queries to q_out.  HBM-bound.
#include <cuda_bf16.h>

#include <cmath>

#include "internal.h"
#include "ptx.cuh"

namespace pa {

__global__ void rope_table_kernel(float* __restrict__ cache, int32_t max_position,
                                  int32_t rotary_dim, double theta) {
  grid_launch_dependents();
  grid_dependency_wait();
  const int half = rotary_dim / 2;
  const int64_t n = static_cast<int64_t>(max_position) * half;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t p = i / half;
    const int k = static_cast<int>(i % half);
    const double f = pow(theta, -2.0 * k / rotary_dim);
    const double a = static_cast<double>(p) * f;
    cache[p * rotary_dim + k] = static_cast<float>(cos(a));
    cache[p * rotary_dim + half + k] = static_cast<float>(sin(a));
  }
}

template <typename T>
struct Chunk;  // 16 bytes of T, as floats
template <>
struct Chunk<float> {
  static constexpr int E = 4;
  static __device__ __forceinline__ void load(const void* p, float (&x)[4]) {
    const float4 v = *static_cast<const float4*>(p);
    x[0] = v.x, x[1] = v.y, x[2] = v.z, x[3] = v.w;
  }
  static __device__ __forceinline__ void store(void* p, const float (&x)[4]) {
    *static_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
};
template <>
struct Chunk<__nv_bfloat16> {
  static constexpr int E = 8;
  static __device__ __forceinline__ void load(const void* p, float (&x)[8]) {
    const uint4 v = *static_cast<const uint4*>(p);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      x[2 * j] = f.x, x[2 * j + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void store(void* p, const float (&x)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = pack_bf16x2(x[2 * j], x[2 * j + 1]);
    *static_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};

struct RopeArgs {
  const void* q_in;
  const void* k;
  const void* v;
  int64_t q_stride, kv_stride;  // elements
  void* q_out;
  void* kc;
  void* vc;
  const int64_t* positions;
  const int64_t* slots;
  const float* cs;
  int32_t max_position, rot;
  int64_t num_tokens;
  int32_t hq, hkv, d;
  int64_t num_slots;
  int32_t* err;
};

// A CTA walks tokens (grid-stride); its threads walk the token's tasks: one
// 16-byte chunk -- or, split-half pairing, one chunk of each half -- of a Q or
// K row (TR per row), then one chunk per V row.  The token's position, slot
// and cos/sin row are shared by the CTA; index arithmetic stays 32-bit.
template <typename T, bool NEOX>
__global__ void __launch_bounds__(256) rope_cache_write_kernel(RopeArgs a) {
  grid_launch_dependents();
  grid_dependency_wait();  // positions / slots may come from the previous launch
  using CK = Chunk<T>;
  constexpr int E = CK::E;
  const int half = a.rot / 2;
  const int PT = NEOX ? a.rot / (2 * E) : a.rot / E;  // rotating tasks per row
  const int TR = PT + (a.d - a.rot) / E;              // tasks per Q or K row
  const int CD = a.d / E;                             // chunks per V row
  const int R = a.hq + a.hkv;
  const int per_token = R * TR + a.hkv * CD;
  const T* qin = static_cast<const T*>(a.q_in);
  const T* kin = static_cast<const T*>(a.k);
  const T* vin = static_cast<const T*>(a.v);
  T* qout = static_cast<T*>(a.q_out);
  T* kc = static_cast<T*>(a.kc);
  T* vc = static_cast<T*>(a.vc);
  const int64_t row_kv = static_cast<int64_t>(a.hkv) * a.d;  // pool row of one slot
  for (int64_t t = blockIdx.x; t < a.num_tokens; t += gridDim.x) {
    const int64_t pos = __ldg(a.positions + t);
    const bool pos_ok = pos >= 0 && pos < a.max_position;
    const int64_t slot = __ldg(a.slots + t);
    const bool slot_in = slot < a.num_slots;
    const bool write = pos_ok && slot >= 0 && slot_in;
    if (threadIdx.x == 0 && a.err) {
      if (!pos_ok) atomicOr(a.err, PA_ERRBIT_POS_OOB);
      else if (!slot_in) atomicOr(a.err, PA_ERRBIT_SLOT_OOB);
    }
    const float* crow = a.cs + (pos_ok ? pos : 0) * a.rot;
    const T* qt = qin + t * a.q_stride;
    const T* kt = kin + t * a.kv_stride;
    T* qo = qout + t * a.hq * a.d;
    T* ks = kc + slot * row_kv;
    const int n_tasks = write ? per_token : a.hq * TR;  // K and V only when stored
    for (int rem = threadIdx.x; rem < n_tasks; rem += blockDim.x) {
      if (rem < R * TR) {
        const int row = rem / TR, task = rem - row * TR;
        const T* src = row < a.hq ? qt + row * a.d : kt + (row - a.hq) * a.d;
        T* dst = row < a.hq ? qo + row * a.d : ks + (row - a.hq) * a.d;
        if (task < PT) {
          const int e0 = task * E;
          if (NEOX) {
            float x1[E], x2[E];
            CK::load(src + e0, x1);
            CK::load(src + e0 + half, x2);
#pragma unroll
            for (int j = 0; j < E; ++j) {
              const float c = pos_ok ? __ldg(crow + e0 + j) : 1.f;
              const float s = pos_ok ? __ldg(crow + half + e0 + j) : 0.f;
              const float y1 = x1[j] * c - x2[j] * s;
              const float y2 = x2[j] * c + x1[j] * s;
              x1[j] = y1;
              x2[j] = y2;
            }
            CK::store(dst + e0, x1);
            CK::store(dst + e0 + half, x2);
          } else {
            float x[E];
            CK::load(src + e0, x);
#pragma unroll
            for (int j = 0; j < E / 2; ++j) {
              const float c = pos_ok ? __ldg(crow + e0 / 2 + j) : 1.f;
              const float s = pos_ok ? __ldg(crow + half + e0 / 2 + j) : 0.f;
              const float x1 = x[2 * j], x2 = x[2 * j + 1];
              x[2 * j] = x1 * c - x2 * s;
              x[2 * j + 1] = x2 * c + x1 * s;
            }
            CK::store(dst + e0, x);
          }
        } else {
          const int e0 = a.rot + (task - PT) * E;
          *reinterpret_cast<uint4*>(dst + e0) = *reinterpret_cast<const uint4*>(src + e0);
        }
      } else {
        const int vr = rem - R * TR;
        const int vrow = vr / CD, e0 = (vr - vrow * CD) * E;
        *reinterpret_cast<uint4*>(vc + slot * row_kv + vrow * a.d + e0) =
            __ldg(reinterpret_cast<const uint4*>(vin + t * a.kv_stride + vrow * a.d + e0));
      }
    }
  }
}

cudaError_t launch_rope_table(float* cache, int32_t max_position, int32_t rotary_dim, double theta,
                              int num_sms, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(max_position) * (rotary_dim / 2);
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, static_cast<int64_t>(num_sms) * 16);
  return launch_pdl<rope_table_kernel>(dim3(static_cast<unsigned>(std::max<int64_t>(blocks, 1))),
                                       dim3(256), 0, s, cache, max_position, rotary_dim, theta);
}

cudaError_t launch_rope_cache_write(const RopeLaunch& l, int num_sms, cudaStream_t s) {
  RopeArgs a{l.q_in, l.k, l.v, l.q_stride, l.kv_stride, l.q_out, l.kc, l.vc, l.positions,
             l.slots, l.cs, l.max_position, l.rot, l.num_tokens, l.hq, l.hkv, l.d, l.num_slots,
             l.err};
  // CTAs walk tokens: 8 per SM resident, a few waves deep
  const int64_t blocks =
      std::max<int64_t>(1, std::min<int64_t>(l.num_tokens, static_cast<int64_t>(num_sms) * 16));
  const dim3 grid(static_cast<unsigned>(blocks)), block(256);
  if (l.dtype == PA_F32)
    return l.neox ? launch_pdl<rope_cache_write_kernel<float, true>>(grid, block, 0, s, a)
                  : launch_pdl<rope_cache_write_kernel<float, false>>(grid, block, 0, s, a);
  return l.neox ? launch_pdl<rope_cache_write_kernel<__nv_bfloat16, true>>(grid, block, 0, s, a)
                : launch_pdl<rope_cache_write_kernel<__nv_bfloat16, false>>(grid, block, 0, s, a);
}

}  // namespace pa
