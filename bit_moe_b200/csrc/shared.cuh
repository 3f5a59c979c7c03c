// shared.cuh -- launchers of the shared expert's 8-bit quantization and FFN.
#pragma once
#include "common.cuh"
namespace bitmoe {
// The shared expert's matrices in 8-bit blocks of 32 (row-major codes,
// fp16 scale per block): gate/up [ffn][hidden], down [hidden][ffn].
struct SharedParams {
  int hidden, ffn;
  const int8_t* gate_q; const uint16_t* gate_d;
  const int8_t* up_q;   const uint16_t* up_d;
  const int8_t* down_q; const uint16_t* down_d;
};
int launch_quantize_weights_q8(const float* w, int64_t rows, int64_t k, int8_t* q, uint16_t* d,
                               cudaStream_t stream);
size_t shared_ws_bytes(int hidden, int ffn, int ntok);
// Most 32-row blocks of the shared ffn that the one-token step computes
// itself (its tagged block outputs live in the layer workspace).
constexpr int kMaxSharedUnits = 64;

// Row r of an 8-bit matrix [rows][k] against activation codes xq [k] with
// scales xd [k/32]: sum over blocks of d_w * d_a * (exact int32 block sum),
// the same value in every lane.
__device__ __forceinline__ float q8_row_dot(const int8_t* __restrict__ q, const uint16_t* __restrict__ d, int k,
                                            const int8_t* __restrict__ xq, const float* __restrict__ xd, int lane) {
  float acc = 0.f;
  for (int j = lane; j < k / kQBlock; j += 32) {
    const int4* wq = reinterpret_cast<const int4*>(q + static_cast<size_t>(j) * kQBlock);
    const int4* aq = reinterpret_cast<const int4*>(xq + static_cast<size_t>(j) * kQBlock);
    const int4 w0 = wq[0], w1 = wq[1], a0 = aq[0], a1 = aq[1];
    int s = __dp4a(w0.x, a0.x, 0);
    s = __dp4a(w0.y, a0.y, s);
    s = __dp4a(w0.z, a0.z, s);
    s = __dp4a(w0.w, a0.w, s);
    s = __dp4a(w1.x, a1.x, s);
    s = __dp4a(w1.y, a1.y, s);
    s = __dp4a(w1.z, a1.z, s);
    s = __dp4a(w1.w, a1.w, s);
    const float sc = __fmul_rn(f16_bits_to_f32(d[j]), xd[j]);
    acc = __fmaf_rn(sc, static_cast<float>(s), acc);
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, m));
  return acc;
}

// q8_row_dot of row gq (scales gd) and of row uq (scales ud) against the same
// activations, with the same per-lane order of blocks and the same arithmetic
// (so the same two values), but every load of both rows for two rounds of
// blocks in flight at once instead of one round trip per block.
__device__ __forceinline__ void q8_row_dot2(const int8_t* __restrict__ gq, const uint16_t* __restrict__ gd,
                                            const int8_t* __restrict__ uq, const uint16_t* __restrict__ ud, int k,
                                            const int8_t* __restrict__ xq, const float* __restrict__ xd, int lane,
                                            float& g_out, float& u_out) {
  const int nbk = k / kQBlock;
  float ga = 0.f, ua = 0.f;
  for (int j0 = 0; j0 < nbk; j0 += 64) {
    int4 gw[2][2], uw[2][2];
    uint16_t gs[2], us[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int j = j0 + lane + 32 * t;
      if (j < nbk) {
        const int4* g4 = reinterpret_cast<const int4*>(gq + static_cast<size_t>(j) * kQBlock);
        const int4* u4 = reinterpret_cast<const int4*>(uq + static_cast<size_t>(j) * kQBlock);
        gw[t][0] = g4[0];
        gw[t][1] = g4[1];
        uw[t][0] = u4[0];
        uw[t][1] = u4[1];
        gs[t] = gd[j];
        us[t] = ud[j];
      }
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int j = j0 + lane + 32 * t;
      if (j < nbk) {
        const int4* aq = reinterpret_cast<const int4*>(xq + static_cast<size_t>(j) * kQBlock);
        const int4 a0 = aq[0], a1 = aq[1];
        int sg = __dp4a(gw[t][0].x, a0.x, 0);
        sg = __dp4a(gw[t][0].y, a0.y, sg);
        sg = __dp4a(gw[t][0].z, a0.z, sg);
        sg = __dp4a(gw[t][0].w, a0.w, sg);
        sg = __dp4a(gw[t][1].x, a1.x, sg);
        sg = __dp4a(gw[t][1].y, a1.y, sg);
        sg = __dp4a(gw[t][1].z, a1.z, sg);
        sg = __dp4a(gw[t][1].w, a1.w, sg);
        int su = __dp4a(uw[t][0].x, a0.x, 0);
        su = __dp4a(uw[t][0].y, a0.y, su);
        su = __dp4a(uw[t][0].z, a0.z, su);
        su = __dp4a(uw[t][0].w, a0.w, su);
        su = __dp4a(uw[t][1].x, a1.x, su);
        su = __dp4a(uw[t][1].y, a1.y, su);
        su = __dp4a(uw[t][1].z, a1.z, su);
        su = __dp4a(uw[t][1].w, a1.w, su);
        ga = __fmaf_rn(__fmul_rn(f16_bits_to_f32(gs[t]), xd[j]), static_cast<float>(sg), ga);
        ua = __fmaf_rn(__fmul_rn(f16_bits_to_f32(us[t]), xd[j]), static_cast<float>(su), ua);
      }
    }
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) {
    ga = __fadd_rn(ga, __shfl_xor_sync(0xffffffffu, ga, m));
    ua = __fadd_rn(ua, __shfl_xor_sync(0xffffffffu, ua, m));
  }
  g_out = ga;
  u_out = ua;
}

// y [ntok][hidden] += the shared expert's FFN of xq, xd; ws holds
// shared_ws_bytes(hidden, ffn, ntok) bytes.
int launch_shared_ffn_add(const SharedParams& S, int ntok, const int8_t* xq, const float* xd, float* y, void* ws,
                          cudaStream_t stream);
}  // namespace bitmoe
