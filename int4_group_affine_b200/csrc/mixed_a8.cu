// mixed_a8.cu - the EdgeRazor mixed ternary / 4-bit layer in weight-activation
// form ("EDGERAZOR 深度解读", section 2.1 矩阵乘法分解, and the 1.88-8-8 / 1.58-8-8
// rows of the weight-activation table in section 3.1):
//   Y[t][o] = s_W[o] * s_X[t] * sum_j Q(W)[o][j] Q(X)[t][j],
// activations quantised to 8 bits per token with the page's symmetric rule at
// n = 8 (s_X = max(max|x| / 127, eps), Q(X) = clip(round(x / s_X), -127, 127)).
// The dot product is integer work (dp4a, exact in int32); the scales come once.
//
// The quantiser writes each token's codes twice, in the byte orders the packed
// weight fields come out of a word in, so a weight word feeds dp4a after a shift
// and a mask with no byte permutes:
//  - for 4-bit rows (8 nibbles per word), each 8-element group as 0 2 4 6 1 3 5 7
//    (w & 0x0F0F0F0F holds elements 0 2 4 6, (w >> 4) & 0x0F0F0F0F elements 1 3 5 7);
//  - for ternary rows (16 2-bit fields per word), each 16-element group as
//    0 4 8 12 1 5 9 13 2 6 10 14 3 7 11 15 ((w >> 2i) & 0x03030303 holds i, 4+i, 8+i, 12+i).
// The stored fields are offset codes (q + 8, q + 1): sum q x = sum field x - offset sum x.
#include "common.cuh"

namespace moeq {
namespace {

constexpr int kAW = 8;   // warps per CTA in the dot kernel (one output row each)
constexpr int kAT = 8;   // tokens per pass of the dot kernel

__device__ __forceinline__ float act_value(const uint16_t* p, int64_t i) { return bf16f(p[i]); }
__device__ __forceinline__ float act_value(const float* p, int64_t i) { return p[i]; }

// One warp per token: scale, codes in natural order (optional), the two permuted copies
// and the code sum.
template <typename Src>
__global__ void act8_kernel(const Src* __restrict__ x, int T, int n, int8_t* __restrict__ qnat,
                            int8_t* __restrict__ q4, int8_t* __restrict__ q2, float* __restrict__ s,
                            int32_t* __restrict__ qsum) {
    const int t = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32, lane = threadIdx.x % 32;
    if (t >= T) return;
    const Src* xr = x + (int64_t)t * n;
    float m = 0.0f;
    for (int j = lane; j < n; j += 32) m = fmaxf(m, fabsf(act_value(xr, j)));
    m = warp_max(m);
    const float sc = fmaxf(__fdiv_rn(m, 127.0f), 1e-5f);
    int sum = 0;
    for (int j = lane; j < n; j += 32) {
        float r = rintf(__fdiv_rn(act_value(xr, j), sc));
        r = fminf(fmaxf(r, -127.0f), 127.0f);
        const int8_t q = (int8_t)r;
        sum += q;
        const int64_t row = (int64_t)t * n;
        if (qnat) qnat[row + j] = q;
        if (q4) {
            const int g = j & ~7, p = j & 7;  // position of element p in its 8-group: 0 2 4 6 1 3 5 7
            q4[row + g + (p >> 1) + ((p & 1) << 2)] = q;
        }
        if (q2) {
            const int g = j & ~15, p = j & 15;  // 0 4 8 12 1 5 9 13 ...: element p at 4 (p % 4) + p / 4
            q2[row + g + ((p & 3) << 2) + (p >> 2)] = q;
        }
    }
    sum = __reduce_add_sync(0xffffffffu, sum);
    if (lane == 0) {
        if (s) s[t] = sc;
        if (qsum) qsum[t] = sum;
    }
}

// sum_j field_j * q_j of one row and kAT tokens (offsets removed by the caller):
// lane-strided over 16-byte pieces of the packed row.
__device__ __forceinline__ void row_dot_a8(const uint32_t* __restrict__ pw, bool four, int in, const int8_t* q4,
                                           const int8_t* q2, int n_act, int t0, int nt, int lane, int (&acc)[kAT]) {
    const int npiece = four ? in / 32 : in / 64;  // 4 words per piece
    const uint4* p4 = reinterpret_cast<const uint4*>(pw);
    for (int c = lane; c < npiece; c += 32) {
        const uint4 wv = p4[c];
        const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
        if (four) {  // piece c: elements 32c .. 32c+31, word k: elements 32c + 8k ..
#pragma unroll
            for (int m = 0; m < kAT; ++m) {
                if (m >= nt) break;
                const int4* xa = reinterpret_cast<const int4*>(q4 + (int64_t)(t0 + m) * n_act + 32 * c);
                const int4 a0 = xa[0], a1 = xa[1];
                const int av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                int s = acc[m];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    s = __dp4a((int)(w[k] & 0x0F0F0F0Fu), av[2 * k], s);
                    s = __dp4a((int)((w[k] >> 4) & 0x0F0F0F0Fu), av[2 * k + 1], s);
                }
                acc[m] = s;
            }
        } else {  // piece c: elements 64c .. 64c+63, word k: elements 64c + 16k ..
#pragma unroll
            for (int m = 0; m < kAT; ++m) {
                if (m >= nt) break;
                const int4* xa = reinterpret_cast<const int4*>(q2 + (int64_t)(t0 + m) * n_act + 64 * c);
                int s = acc[m];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int4 a = xa[k];
                    s = __dp4a((int)(w[k] & 0x03030303u), a.x, s);
                    s = __dp4a((int)((w[k] >> 2) & 0x03030303u), a.y, s);
                    s = __dp4a((int)((w[k] >> 4) & 0x03030303u), a.z, s);
                    s = __dp4a((int)((w[k] >> 6) & 0x03030303u), a.w, s);
                }
                acc[m] = s;
            }
        }
    }
#pragma unroll
    for (int m = 0; m < kAT; ++m) acc[m] = __reduce_add_sync(0xffffffffu, acc[m]);
}

struct A8Args {
    moe_mixed_tensor W, U;  // W: the layer (gate in mode 1); U: up (mode 1 only)
    int G, T;
    const int8_t *q4, *q2;
    const float* sx;
    const int32_t* qsum;
    int mode;                 // 0: y fp32 [T][out]; 1: h = SiLU(W x) * (U x) fp32; 2: y bf16 (+ residual)
    float* yf;
    uint16_t* yb;
    const uint16_t* residual;
};

__global__ void __launch_bounds__(kAW * 32) mixed_a8_kernel(const __grid_constant__ A8Args a) {
    const int o = blockIdx.x * kAW + threadIdx.x / 32, lane = threadIdx.x % 32;
    const int out = a.W.out, in = a.W.in;
    if (o >= out) return;
    const bool four = a.G > 0 && o % a.G == 0;
    const uint32_t* pw = a.W.packed + mixed_row_offset(o, in, a.G);
    const float sw = bf16f(a.W.scales[o]);
    const int off = four ? 8 : 1;
    const uint32_t* pu = a.mode == 1 ? a.U.packed + mixed_row_offset(o, in, a.G) : nullptr;
    const float su = a.mode == 1 ? bf16f(a.U.scales[o]) : 0.0f;
    for (int t0 = 0; t0 < a.T; t0 += kAT) {
        const int nt = min(kAT, a.T - t0);
        int acc[kAT], accu[kAT];
#pragma unroll
        for (int m = 0; m < kAT; ++m) acc[m] = accu[m] = 0;
        row_dot_a8(pw, four, in, a.q4, a.q2, in, t0, nt, lane, acc);
        if (pu) row_dot_a8(pu, four, in, a.q4, a.q2, in, t0, nt, lane, accu);
        if (lane < nt) {
            int av = 0, au = 0;
#pragma unroll
            for (int m = 0; m < kAT; ++m)
                if (m == lane) {
                    av = acc[m];
                    au = accu[m];
                }
            const int t = t0 + lane;
            const float st = a.sx[t];
            const float v = (float)(av - off * a.qsum[t]) * sw * st;
            if (a.mode == 0) {
                a.yf[(int64_t)t * out + o] = v;
            } else if (a.mode == 1) {
                const float u = (float)(au - off * a.qsum[t]) * su * st;
                a.yf[(int64_t)t * out + o] = silu(v) * u;
            } else {
                const float r = a.residual ? bf16f(a.residual[(int64_t)t * out + o]) : 0.0f;
                a.yb[(int64_t)t * out + o] = f2bf16(r + v);
            }
        }
    }
}

}  // namespace

cudaError_t launch_act8(const uint16_t* xb, const float* xf, int T, int n, int8_t* qnat, int8_t* q4, int8_t* q2,
                        float* s, int32_t* qsum, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int warps = 4;
    if (xb)
        act8_kernel<uint16_t><<<(T + warps - 1) / warps, warps * 32, 0, st>>>(xb, T, n, qnat, q4, q2, s, qsum);
    else
        act8_kernel<float><<<(T + warps - 1) / warps, warps * 32, 0, st>>>(xf, T, n, qnat, q4, q2, s, qsum);
    return cudaGetLastError();
}

cudaError_t launch_mixed_a8(const moe_mixed_tensor& W, const moe_mixed_tensor* U, int G, const int8_t* q4,
                            const int8_t* q2, const float* sx, const int32_t* qsum, int T, int mode, float* yf,
                            uint16_t* yb, const uint16_t* residual, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    A8Args a;
    a.W = W;
    a.U = U ? *U : W;
    a.G = G;
    a.T = T;
    a.q4 = q4;
    a.q2 = q2;
    a.sx = sx;
    a.qsum = qsum;
    a.mode = mode;
    a.yf = yf;
    a.yb = yb;
    a.residual = residual;
    mixed_a8_kernel<<<(W.out + kAW - 1) / kAW, kAW * 32, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moeq
