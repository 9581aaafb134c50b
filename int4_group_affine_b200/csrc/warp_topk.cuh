// warp_topk.cuh - one warp's softmax + top-K + renormalisation over E <= 512 logits.
#pragma once

#include "common.cuh"

namespace moeq {

// z: the token's logits (E entries; kL2: global memory written by other CTAs,
// read from L2; otherwise shared memory).  Writes idx[0..K) in
// descending logit order (equal logits: lower expert first) and w = p / sum of
// the chosen p, on every lane.  Returns false if no finite logit was found.
template <bool kL2>
__device__ __forceinline__ void warp_topk(const float* z, int E, int K, int* idx, float* w) {
    constexpr int kPer = MOEQ_MAX_EXPERTS / 32;
    const int lane = threadIdx.x % 32;
    float zv[kPer], pv[kPer];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        zv[i] = e < E ? (kL2 ? __ldcg(z + e) : z[e]) : -INFINITY;
        m = fmaxf(m, zv[i]);
    }
    m = warp_max(m);
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        pv[i] = e < E ? expf(zv[i] - m) : 0.0f;
        s += pv[i];
    }
    s = warp_sum(s);
    uint32_t taken = 0;
    float psum = 0.0f;
    for (int k = 0; k < K; ++k) {
        float bz = -INFINITY;
        int be = 0x7fffffff, bi = -1;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u) && (bi < 0 || zv[i] > bz)) {
                bz = zv[i];
                be = e;
                bi = i;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float oz = __shfl_xor_sync(0xffffffffu, bz, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (oz > bz || (oz == bz && oe < be)) {
                bz = oz;
                be = oe;
            }
        }
        if (be >= E) be = 0;  // only reachable with NaN logits
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        float pe = 0.0f;
#pragma unroll
        for (int i = 0; i < kPer; ++i)
            if (lane + 32 * i == be) pe = pv[i];
        pe = __shfl_sync(0xffffffffu, pe, be & 31) / s;
        idx[k] = be;
        w[k] = pe;
        psum += pe;
    }
    for (int k = 0; k < K; ++k) w[k] /= psum;
}

}  // namespace moeq
