// router.cu - a1/a2: 8-bit group-affine router and shared-expert gate logits,
// then softmax, top-K (ties to the lower index) and renormalisation.
#include "common.cuh"

namespace moeq {
namespace {

constexpr int kRouterWarps = 8;
constexpr int kRowsPerWarp = 4;
constexpr int kRouterRows = kRouterWarps * kRowsPerWarp;  // rows per CTA
constexpr int kRouterTokMax = 8;                          // tokens per CTA (H <= 6144)

// Grid (ceil(R / 32), ceil(T / 8)), R = E (+1 for the shared gate, stored in gs).
// Each warp walks one int8 row with 16-byte loads (4 words = 16 weights per lane
// per step), dequantises w = s*q + b in registers and dots it with up to 8
// token rows staged in shared memory as fp32.
template <int kRouterTok>
__global__ void __launch_bounds__(kRouterWarps * 32)
router_logits_kernel(const uint16_t* __restrict__ x, moe_qtensor router, moe_qtensor sgate, int has_sgate,
                     const float* __restrict__ logit_bias, int T, int H, int E, float* __restrict__ logits,
                     float* __restrict__ gs) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);  // [kRouterTok][H]
    const int t0 = blockIdx.y * kRouterTok;
    const int nt = min(kRouterTok, T - t0);
    for (int i = threadIdx.x; i < kRouterTok * H; i += blockDim.x) {
        const int tt = i / H, j = i % H;
        xs[i] = tt < nt ? bf16f(x[(int64_t)(t0 + tt) * H + j]) : 0.0f;
    }
    __syncthreads();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int R = E + (has_sgate ? 1 : 0);
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int row = blockIdx.x * kRouterRows + warp * kRowsPerWarp + rr;
        if (row >= R) break;
        const moe_qtensor& m = row < E ? router : sgate;
        const int r = row < E ? row : 0;
        const int words = H / 4;
        const int ng = H / m.group;
        const uint4* pw = reinterpret_cast<const uint4*>(m.packed + (int64_t)r * words);
        const uint16_t* sc = m.scales + (int64_t)r * ng;
        const uint16_t* bi = m.biases + (int64_t)r * ng;
        float acc[kRouterTok];
#pragma unroll
        for (int tt = 0; tt < kRouterTok; ++tt) acc[tt] = 0.0f;
        for (int v = lane; v < words / 4; v += 32) {
            const uint4 q4 = pw[v];
            const uint32_t qs[4] = {q4.x, q4.y, q4.z, q4.w};
            const int j0 = v * 16;  // first element covered by this 16-byte vector
            const int g = j0 / m.group;
            const float s = bf16f(sc[g]), b = bf16f(bi[g]);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float wv[4];
#pragma unroll
                for (int f = 0; f < 4; ++f) wv[f] = __fmaf_rn(s, u2f_small((qs[k] >> (8 * f)) & 0xFFu), b);
#pragma unroll
                for (int tt = 0; tt < kRouterTok; ++tt) {
                    const float4 xv = *reinterpret_cast<const float4*>(&xs[tt * H + j0 + 4 * k]);
                    acc[tt] = fmaf(wv[0], xv.x, acc[tt]);
                    acc[tt] = fmaf(wv[1], xv.y, acc[tt]);
                    acc[tt] = fmaf(wv[2], xv.z, acc[tt]);
                    acc[tt] = fmaf(wv[3], xv.w, acc[tt]);
                }
            }
        }
#pragma unroll
        for (int tt = 0; tt < kRouterTok; ++tt) acc[tt] = warp_sum(acc[tt]);
        if (lane < nt) {
            float v = 0.0f;
#pragma unroll
            for (int tt = 0; tt < kRouterTok; ++tt)
                if (tt == lane) v = acc[tt];
            if (row < E) logits[(int64_t)(t0 + lane) * E + row] = v + (logit_bias ? logit_bias[row] : 0.0f);
            else gs[t0 + lane] = v;
        }
    }
}

// The shared-expert gate alone (the routed logits come from the tensor cores): one warp
// per token dots the int8 row (H bytes, read from L2) with the token's x, 16 weights per
// lane and step in 16-byte pieces, every piece of a step in flight together;
// w = s*q + b in fp32 as in router_logits_kernel.
__global__ void __launch_bounds__(256) sgate_logits_kernel(const uint16_t* __restrict__ x, moe_qtensor sg, int T,
                                                           int H, float* __restrict__ gs) {
    const int t = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
    if (t >= T) return;
    const int nv = H / 16;
    const uint4* pw = reinterpret_cast<const uint4*>(sg.packed);
    const uint4* px = reinterpret_cast<const uint4*>(x + (int64_t)t * H);
    float acc = 0.0f;
    for (int v0 = lane; v0 < nv; v0 += 32 * 4) {
        uint4 q[4], xa[4], xb[4];
        float s[4], b[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int v = v0 + 32 * j;
            if (v < nv) {
                q[j] = pw[v];
                xa[j] = px[2 * v];
                xb[j] = px[2 * v + 1];
                const int g = v * 16 / sg.group;
                s[j] = bf16f(sg.scales[g]);
                b[j] = bf16f(sg.biases[g]);
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (v0 + 32 * j >= nv) break;
            const uint32_t qs[4] = {q[j].x, q[j].y, q[j].z, q[j].w};
            const uint32_t xw[8] = {xa[j].x, xa[j].y, xa[j].z, xa[j].w, xb[j].x, xb[j].y, xb[j].z, xb[j].w};
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float w = __fmaf_rn(s[j], u2f_small((qs[e / 4] >> (8 * (e % 4))) & 0xFFu), b[j]);
                const float xv = __uint_as_float(e % 2 ? xw[e / 2] & 0xFFFF0000u : xw[e / 2] << 16);
                acc = fmaf(w, xv, acc);
            }
        }
    }
    acc = warp_sum(acc);
    if (lane == 0) gs[t] = acc;
}

// One warp per token: softmax over E logits, K rounds of warp argmax.
__global__ void topk_kernel(const float* __restrict__ logits, const float* gs, int has_sgate, int T,
                            int E, int K, int32_t* __restrict__ idx, float* __restrict__ w,
                            float* sg) {  // gs and sg may alias (moe_router_topk)
    const int warps = blockDim.x / 32;
    const int t = blockIdx.x * warps + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (t >= T) return;
    constexpr int kPer = MOEQ_MAX_EXPERTS / 32;
    float z[kPer], p[kPer];
    const float* zr = logits + (int64_t)t * E;
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        z[i] = e < E ? zr[e] : -INFINITY;
        m = fmaxf(m, z[i]);
    }
    m = warp_max(m);
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        p[i] = e < E ? expf(z[i] - m) : 0.0f;
        s += p[i];
    }
    s = warp_sum(s);
    uint32_t taken = 0;  // bit i: slot i of this lane already chosen
    float psel[MOEQ_MAX_TOPK];
    int esel[MOEQ_MAX_TOPK];
    float psum = 0.0f;
    for (int k = 0; k < K; ++k) {
        float bz = -INFINITY;
        int be = 0x7fffffff, bi = -1;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u) && (bi < 0 || z[i] > bz)) {
                bz = z[i];
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
            if (lane + 32 * i == be) pe = p[i];
        pe = __shfl_sync(0xffffffffu, pe, be & 31) / s;
        psel[k] = pe;
        esel[k] = be;
        psum += pe;
    }
    if (lane == 0) {
        for (int k = 0; k < K; ++k) {
            idx[(int64_t)t * K + k] = esel[k];
            w[(int64_t)t * K + k] = psel[k] / psum;
        }
        if (sg) sg[t] = has_sgate ? 1.0f / (1.0f + expf(-gs[t])) : 1.0f;
    }
}

}  // namespace

cudaError_t launch_router_logits(const uint16_t* x, const moe_qtensor& router, const moe_qtensor* sgate,
                                 const float* logit_bias, int T, int H, int E, float* logits, float* gs,
                                 cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int has = (sgate && sgate->packed) ? 1 : 0;
    const int R = E + has;
    moe_qtensor sg = has ? *sgate : router;
    const int tok = H <= 6144 ? kRouterTokMax : kRouterTokMax / 2;
    dim3 grid((R + kRouterRows - 1) / kRouterRows, (T + tok - 1) / tok);
    const size_t smem = (size_t)tok * H * sizeof(float);
    if (tok == kRouterTokMax) {
        static int cached = 0;
        cudaError_t e = ensure_smem((const void*)router_logits_kernel<kRouterTokMax>, smem, cached);
        if (e != cudaSuccess) return e;
        router_logits_kernel<kRouterTokMax>
            <<<grid, kRouterWarps * 32, smem, s>>>(x, router, sg, has, logit_bias, T, H, E, logits, gs);
    } else {
        static int cached = 0;
        cudaError_t e = ensure_smem((const void*)router_logits_kernel<kRouterTokMax / 2>, smem, cached);
        if (e != cudaSuccess) return e;
        router_logits_kernel<kRouterTokMax / 2>
            <<<grid, kRouterWarps * 32, smem, s>>>(x, router, sg, has, logit_bias, T, H, E, logits, gs);
    }
    return cudaGetLastError();
}

cudaError_t launch_sgate_logits(const uint16_t* x, const moe_qtensor& sgate, int T, int H, float* gs,
                                cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    sgate_logits_kernel<<<(T + 7) / 8, 256, 0, s>>>(x, sgate, T, H, gs);
    return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, const float* gs, bool has_sgate, int T, int E, int K, int32_t* idx,
                        float* w, float* sg, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int warps = 4;
    topk_kernel<<<(T + warps - 1) / warps, warps * 32, 0, s>>>(logits, gs, has_sgate ? 1 : 0, T, E, K, idx, w, sg);
    return cudaGetLastError();
}

namespace {

__global__ void select_kernel(const float* __restrict__ logits, const float* gs, int has_sgate,
                              const int32_t* __restrict__ sel, int T, int E, int K, int32_t* __restrict__ idx,
                              float* __restrict__ w, float* sg, int32_t* status) {
    const int warps = blockDim.x / 32;
    const int t = blockIdx.x * warps + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (t >= T) return;
    bool bad = false;
    const int e = select_entry(sel + (int64_t)t * K, K, E, lane, &bad);
    if (bad && lane == 0) raise_status(status, MOE_ERR_DEVICE_INDEX);
    const float z = e >= 0 ? logits[(int64_t)t * E + e] : -INFINITY;
    const float m = warp_max(z);
    const float ev = e >= 0 ? expf(z - m) : 0.0f;
    const float sum = warp_sum(ev);
    if (lane < K) {
        idx[(int64_t)t * K + lane] = e;
        w[(int64_t)t * K + lane] = ev / sum;
    }
    if (lane == 0 && sg) sg[t] = has_sgate ? 1.0f / (1.0f + expf(-gs[t])) : 1.0f;
}

}  // namespace

cudaError_t launch_select(const float* logits, const float* gs, bool has_sgate, const int32_t* sel, int T, int E,
                          int K, int32_t* idx, float* w, float* sg, int32_t* status, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int warps = 4;
    select_kernel<<<(T + warps - 1) / warps, warps * 32, 0, s>>>(logits, gs, has_sgate ? 1 : 0, sel, T, E, K, idx, w,
                                                                 sg, status);
    return cudaGetLastError();
}

}  // namespace moeq
