// mixed.cu - a7: EdgeRazor mixed ternary / 4-bit weight-only GEMV/GEMM.
// y_o = s_o * sum_j q_oj x_j: the integer codes are dotted with the activations and
// the per-row scale is applied once at the end (the weight-only form of the EdgeRazor
// matmul decomposition).  Up to a few tokens on CUDA cores (below); batches on warp-level
// tensor-core tiles (further down).
//
// Row layout: super-groups of G rows, the first 4-bit (in/8 words, nibble q+8),
// the rest ternary (in/16 words, 2-bit field q+1).  A warp owns one output row
// and streams it with 16-byte loads: a vector is 32 elements of a 4-bit row or
// 64 elements of a ternary row.  Codes are offset (q+8, q+1), so the kernels
// dot the raw field with x and subtract offset * sum(x) per 32-element chunk.
#include "common.cuh"

namespace moeq {
namespace {

constexpr int kMT = 8;      // tokens per shared-memory chunk (the largest instantiation)
constexpr int kMWarps = 8;  // warps (rows) per CTA

__device__ __forceinline__ int mswz(int j) {
    const int c = j >> 5;
    return (c << 5) | (((j & 31) + ((c & 7) << 2)) & 31);
}

// Stage the nt live token rows (of at most MT) of length n into swizzled fp32 shared
// memory with 32-element chunk sums.  Rows at 16-byte aligned addresses come in 16-byte
// pieces (8 bf16 or 4 fp32 values, one per thread and step; the lanes of a chunk add
// their sums with shuffles); other rows value by value.
template <int MT, typename Src>
__device__ void mstage(float* xs, float* xsum, const Src* src, int ld, int t0, int nt, int n) {
    constexpr int kE = 16 / (int)sizeof(Src);  // values per 16-byte piece
    constexpr int kL = 32 / kE;                // pieces (lanes) per 32-value chunk
    const Src* base = src + (int64_t)t0 * ld;
    const bool vec = ((((uintptr_t)base) | ((uintptr_t)ld * sizeof(Src))) & 15) == 0;
    if (vec) {
        const int per = n / kE, total = nt * per, lim = (total + 31) / 32 * 32;
        for (int i = threadIdx.x; i < lim; i += blockDim.x) {
            const bool live = i < total;
            const int tt = live ? i / per : 0, q = live ? i % per : 0;
            float f[kE];
            if (live) {
                const uint4 u = reinterpret_cast<const uint4*>(base + (int64_t)tt * ld)[q];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
                if constexpr (kE == 8) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        f[2 * k] = __uint_as_float(w[k] << 16);
                        f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k) f[k] = __uint_as_float(w[k]);
                }
            } else {
#pragma unroll
                for (int k = 0; k < kE; ++k) f[k] = 0.0f;
            }
            const int c = q / kL, o = (q % kL) * kE, rot = (c & 7) << 2;
            float sm = 0.0f;
#pragma unroll
            for (int k = 0; k < kE; ++k) sm += f[k];
#pragma unroll
            for (int x = 1; x < kL; x <<= 1) sm += __shfl_xor_sync(0xffffffffu, sm, x);
            if (live) {
                float* d = xs + tt * n + (c << 5);
#pragma unroll
                for (int k = 0; k < kE; k += 4)
                    *reinterpret_cast<float4*>(d + ((o + k + rot) & 31)) = make_float4(f[k], f[k + 1], f[k + 2], f[k + 3]);
                if (q % kL == 0) xsum[tt * (n / 32) + c] = sm;
            }
        }
        __syncthreads();
        return;
    }
    for (int i = threadIdx.x; i < nt * n; i += blockDim.x) {
        const int tt = i / n, j = i % n;
        float v;
        if constexpr (sizeof(Src) == 2) v = bf16f(base[(int64_t)tt * ld + j]);
        else v = base[(int64_t)tt * ld + j];
        xs[tt * n + mswz(j)] = v;
    }
    __syncthreads();
    const int nc = n / 32;
    for (int i = threadIdx.x; i < nt * nc; i += blockDim.x) {
        const int tt = i / nc, c = i % nc;
        float sm = 0.0f;
        for (int f = 0; f < 32; ++f) sm += xs[tt * n + (c << 5) + f];
        xsum[i] = sm;
    }
    __syncthreads();
}

// Dot of 32 consecutive code fields (bits = 4 or 2, stored in `nw` words) with
// chunk c of each of the nt staged tokens; subtracts offset * chunk sum.
template <int BITS, int MT>
__device__ __forceinline__ void code_chunk(const uint32_t* w, int c, float offset, const float* xs, const float* xsum,
                                           int n, int nt, float* acc) {
    constexpr int kPer = 32 / BITS;  // fields per word
    constexpr uint32_t kMask = (1u << BITS) - 1u;
    float qf[32];
#pragma unroll
    for (int f = 0; f < 32; ++f) qf[f] = u2f_small((w[f / kPer] >> (BITS * (f % kPer))) & kMask);
    const int rot = (c & 7) << 2;
#pragma unroll
    for (int tt = 0; tt < MT; ++tt) {
        if (tt >= nt) break;
        const float* xr = xs + tt * n + (c << 5);
        float a = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 xv = *reinterpret_cast<const float4*>(xr + ((4 * q + rot) & 31));
            a = fmaf(qf[4 * q + 0], xv.x, a);
            a = fmaf(qf[4 * q + 1], xv.y, a);
            a = fmaf(qf[4 * q + 2], xv.z, a);
            a = fmaf(qf[4 * q + 3], xv.w, a);
        }
        acc[tt] += fmaf(-offset, xsum[tt * (n / 32) + c], a);
    }
}

// sum_j q_oj x[tt][j] for one row, accumulated per lane (caller reduces).
template <int MT>
__device__ __forceinline__ void mixed_row(const moe_mixed_tensor& W, int G, int o, const float* xs, const float* xsum,
                                          int nt, float* acc, int lane) {
    const int n = W.in;
    const uint32_t* pw = W.packed + mixed_row_offset(o, n, G);
    if (G > 0 && o % G == 0) {
        const uint4* v4 = reinterpret_cast<const uint4*>(pw);
        for (int c = lane; c < n / 32; c += 32) {
            const uint4 q = v4[c];
            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
            code_chunk<4, MT>(w, c, 8.0f, xs, xsum, n, nt, acc);
        }
    } else {
        const uint4* v4 = reinterpret_cast<const uint4*>(pw);
        for (int v = lane; v < n / 64; v += 32) {
            const uint4 q = v4[v];
            const uint32_t w0[2] = {q.x, q.y}, w1[2] = {q.z, q.w};
            code_chunk<2, MT>(w0, 2 * v, 1.0f, xs, xsum, n, nt, acc);
            code_chunk<2, MT>(w1, 2 * v + 1, 1.0f, xs, xsum, n, nt, acc);
        }
    }
}

// MT: tokens per shared-memory chunk of this instantiation (T is walked in chunks of MT).
template <int MT>
__global__ void __launch_bounds__(kMWarps * 32)
mixed_linear_kernel(moe_mixed_tensor W, int G, const uint16_t* __restrict__ x, int T, float* __restrict__ y) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);
    float* xsum = xs + MT * W.in;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int o = blockIdx.x * kMWarps + warp;
    for (int t0 = 0; t0 < T; t0 += MT) {
        const int nt = min(MT, T - t0);
        __syncthreads();
        mstage<MT>(xs, xsum, x, W.in, t0, nt, W.in);
        if (o >= W.out) continue;
        float acc[MT];
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) acc[tt] = 0.0f;
        mixed_row<MT>(W, G, o, xs, xsum, nt, acc, lane);
        const float s = bf16f(W.scales[o]);
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) {
            if (tt >= nt) break;
            const float v = warp_sum(acc[tt]);
            if (lane == 0) y[(int64_t)(t0 + tt) * W.out + o] = s * v;
        }
    }
}

template <int MT>
__global__ void __launch_bounds__(kMWarps * 32)
mixed_gate_up_kernel(moe_mixed_tensor Wg, moe_mixed_tensor Wu, int G, const uint16_t* __restrict__ x, int T,
                     float* __restrict__ h) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);
    float* xsum = xs + MT * Wg.in;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int o = blockIdx.x * kMWarps + warp;
    for (int t0 = 0; t0 < T; t0 += MT) {
        const int nt = min(MT, T - t0);
        __syncthreads();
        mstage<MT>(xs, xsum, x, Wg.in, t0, nt, Wg.in);
        if (o >= Wg.out) continue;
        float ag[MT], au[MT];
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) ag[tt] = au[tt] = 0.0f;
        mixed_row<MT>(Wg, G, o, xs, xsum, nt, ag, lane);
        mixed_row<MT>(Wu, G, o, xs, xsum, nt, au, lane);
        const float sg = bf16f(Wg.scales[o]), su = bf16f(Wu.scales[o]);
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) {
            if (tt >= nt) break;
            const float g = sg * warp_sum(ag[tt]);
            const float u = su * warp_sum(au[tt]);
            if (lane == 0) h[(int64_t)(t0 + tt) * Wg.out + o] = silu(g) * u;
        }
    }
}

template <int MT>
__global__ void __launch_bounds__(kMWarps * 32)
mixed_down_kernel(moe_mixed_tensor Wd, int G, const float* __restrict__ h, int T, const uint16_t* __restrict__ res,
                  uint16_t* __restrict__ y) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);
    float* xsum = xs + MT * Wd.in;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int o = blockIdx.x * kMWarps + warp;
    for (int t0 = 0; t0 < T; t0 += MT) {
        const int nt = min(MT, T - t0);
        __syncthreads();
        mstage<MT>(xs, xsum, h, Wd.in, t0, nt, Wd.in);
        if (o >= Wd.out) continue;
        float acc[MT];
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) acc[tt] = 0.0f;
        mixed_row<MT>(Wd, G, o, xs, xsum, nt, acc, lane);
        const float s = bf16f(Wd.scales[o]);
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) {
            if (tt >= nt) break;
            float v = s * warp_sum(acc[tt]);
            if (lane == 0) {
                const int64_t i = (int64_t)(t0 + tt) * Wd.out + o;
                if (res) v += bf16f(res[i]);
                y[i] = f2bf16(v);
            }
        }
    }
}

size_t stage_bytes(int n, int mt) { return (size_t)mt * n * sizeof(float) + (size_t)mt * (n / 32) * sizeof(float); }

int mt_for(int T) { return T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : kMT; }

// ------------------------------------------------------------------ batches: mma.sync tiles
// From kQMinTokens tokens on, the same products on the tensor cores with warp-level
// mma.sync (m16n8k16, bf16 in, fp32 accumulate): the codes are small integers, exact in
// bf16, so the tile is q (not s q) and the per-row scale is applied once at the end.  A CTA
// of kQWarps warps owns 16 output rows; warp w the K slice [w n/kQWarps, (w+1) n/kQWarps);
// each lane builds its A fragment straight from its two rows' packed words.  The inputs of
// up to kQTok tokens per pass are staged as bf16 (an fp32 input as two bf16 planes hi and
// lo = bf16(v - hi), two MMAs into one accumulator, about 16 bits of each value); the
// warps' partial tiles are added in fixed order in shared memory.  The K loop of a warp is
// only n/kQWarps long and N is at most 16 tokens: the kernel is bound by issue and latency,
// not by the tensor pipe, which is why the warp-level MMA serves here.
constexpr int kQWarps = 16;
constexpr int kQTok = 16;        // tokens per pass: two n-tiles of 8
constexpr int kQMinTokens = 4;

enum QMode { kQLinear = 0, kQGateUp = 1, kQDown = 2 };

struct QArgs {
    moe_mixed_tensor W0, W1;  // the matrix (gate for kQGateUp), and up
    int G, T;
    const uint16_t* xb;       // bf16 inputs [T][n] (linear, gate/up)
    const float* xf;          // fp32 inputs [T][n] (down)
    float* yf;                // linear: [T][out]; gate/up: h [T][out]
    uint16_t* yb;             // down: bf16 [T][out]
    const uint16_t* res;      // down: residual [T][out] or null
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two code fields of t (bits 0.. and bits `step`.., `mask` wide) as the bf16 pair
// (f0 - off, f1 - off), low half first: the fields go into the mantissa of bf16 128.0
// (bits 0x4300), whose last mantissa bit counts 1, and 128 + off is subtracted exactly.
template <int kStep, uint32_t kMask>
__device__ __forceinline__ uint32_t code_pair(uint32_t t, __nv_bfloat162 sub) {
    const uint32_t v = (t & kMask) | ((t << (16 - kStep)) & (kMask << 16)) | 0x43004300u;
    __nv_bfloat162 p = *reinterpret_cast<const __nv_bfloat162*>(&v);
    p = __hsub2(p, sub);
    return *reinterpret_cast<const uint32_t*>(&p);
}

// This lane's A-fragment pairs of one row for the 4 k16 blocks of a 64-wide K superblock:
// frag[kb][0] = K (2c, 2c+1), frag[kb][1] = K (2c+8, 2c+9) of block kb (c = lane % 4).
__device__ __forceinline__ void row_frags(const uint32_t* pw, bool four, int k64, int c, uint32_t (&frag)[4][2]) {
    if (four) {  // 8 words of 8 nibbles (value + 8)
        const uint4* v4 = reinterpret_cast<const uint4*>(pw) + k64 * 2;
        const uint4 u0 = v4[0], u1 = v4[1];
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        const __nv_bfloat162 sub = __floats2bfloat162_rn(136.0f, 136.0f);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            frag[kb][0] = code_pair<4, 0xFu>(w[2 * kb] >> (8 * c), sub);
            frag[kb][1] = code_pair<4, 0xFu>(w[2 * kb + 1] >> (8 * c), sub);
        }
    } else {  // 4 words of 16 two-bit fields (value + 1)
        const uint4 u = reinterpret_cast<const uint4*>(pw)[k64];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        const __nv_bfloat162 sub = __floats2bfloat162_rn(129.0f, 129.0f);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            frag[kb][0] = code_pair<2, 0x3u>(w[kb] >> (4 * c), sub);
            frag[kb][1] = code_pair<2, 0x3u>(w[kb] >> (4 * c + 16), sub);
        }
    }
}

__device__ __forceinline__ uint32_t bits_of(__nv_bfloat162 v) { return *reinterpret_cast<const uint32_t*>(&v); }

template <int kMode>
__global__ void __launch_bounds__(kQWarps * 32) mixed_mma_kernel(const __grid_constant__ QArgs a) {
    constexpr int kPlanes = kMode == kQDown ? 2 : 1;
    constexpr int kMats = kMode == kQGateUp ? 2 : 1;
    extern __shared__ float4 smem_f4[];
    const int n = a.W0.in, P = n + 8, out = a.W0.out;
    uint16_t* planes = reinterpret_cast<uint16_t*>(smem_f4);  // [kPlanes][kQTok][P] bf16
    float* part = reinterpret_cast<float*>(planes + (size_t)kPlanes * kQTok * P);  // [kQWarps][kMats][16][kQTok]
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, g = lane >> 2, c = lane & 3;
    const int r0 = blockIdx.x * 16, ks = n / kQWarps;
    const uint32_t* pw[kMats][2];
    bool four[kMats][2];
#pragma unroll
    for (int m = 0; m < kMats; ++m)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const moe_mixed_tensor& M = m ? a.W1 : a.W0;
            const int row = r0 + g + 8 * rr;
            pw[m][rr] = M.packed + mixed_row_offset(row, n, a.G);
            four[m][rr] = a.G > 0 && row % a.G == 0;
        }
    for (int t0 = 0; t0 < a.T; t0 += kQTok) {
        const int nt = min(kQTok, a.T - t0);
        __syncthreads();  // the previous pass is done with the planes and the partial tiles
        if constexpr (kMode == kQDown) {  // fp32 inputs: hi and lo planes, 4 values per piece
            const int per = n / 4, total = kQTok * per;
            for (int i0 = threadIdx.x; i0 < total; i0 += 4 * blockDim.x) {
                float4 v[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = i0 + j * blockDim.x, tok = i / per;
                    v[j] = i < total && tok < nt ? reinterpret_cast<const float4*>(a.xf + (int64_t)(t0 + tok) * n)[i % per]
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = i0 + j * blockDim.x;
                    if (i >= total) break;
                    const int tok = i / per, q = i % per;
                    const __nv_bfloat162 h0 = __floats2bfloat162_rn(v[j].x, v[j].y);
                    const __nv_bfloat162 h1 = __floats2bfloat162_rn(v[j].z, v[j].w);
                    const float2 f0 = __bfloat1622float2(h0), f1 = __bfloat1622float2(h1);
                    const __nv_bfloat162 l0 = __floats2bfloat162_rn(v[j].x - f0.x, v[j].y - f0.y);
                    const __nv_bfloat162 l1 = __floats2bfloat162_rn(v[j].z - f1.x, v[j].w - f1.y);
                    reinterpret_cast<uint2*>(planes + (size_t)tok * P)[q] = make_uint2(bits_of(h0), bits_of(h1));
                    reinterpret_cast<uint2*>(planes + (size_t)(kQTok + tok) * P)[q] = make_uint2(bits_of(l0), bits_of(l1));
                }
            }
        } else {  // bf16 inputs, 8 values per piece
            const int per = n / 8, total = kQTok * per;
            for (int i0 = threadIdx.x; i0 < total; i0 += 4 * blockDim.x) {
                uint4 v[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = i0 + j * blockDim.x, tok = i / per;
                    v[j] = i < total && tok < nt ? reinterpret_cast<const uint4*>(a.xb + (int64_t)(t0 + tok) * n)[i % per]
                                                 : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = i0 + j * blockDim.x;
                    if (i >= total) break;
                    reinterpret_cast<uint4*>(planes + (size_t)(i / per) * P)[i % per] = v[j];
                }
            }
        }
        __syncthreads();
        float acc[kMats][2][4];
#pragma unroll
        for (int m = 0; m < kMats; ++m)
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[m][j][e] = 0.0f;
        for (int s = 0; s < ks / 64; ++s) {
            const int k64 = warp * (ks / 64) + s;  // 64-wide K superblock of the row
            uint32_t fa[kMats][2][4][2];
#pragma unroll
            for (int m = 0; m < kMats; ++m)
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) row_frags(pw[m][rr], four[m][rr], k64, c, fa[m][rr]);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                const int k = k64 * 64 + 16 * kb + 2 * c;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
#pragma unroll
                    for (int pl = 0; pl < kPlanes; ++pl) {
                        const uint16_t* bp = planes + (size_t)(pl * kQTok + 8 * j + g) * P + k;
                        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(bp);
                        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(bp + 8);
#pragma unroll
                        for (int m = 0; m < kMats; ++m)
                            mma_bf16_16816(acc[m][j], fa[m][0][kb][0], fa[m][1][kb][0], fa[m][0][kb][1], fa[m][1][kb][1],
                                           b0, b1);
                    }
                }
            }
        }
        // this warp's partial tile: rows g, g + 8, tokens 8 j + 2 c, + 1
#pragma unroll
        for (int m = 0; m < kMats; ++m)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float* pp = part + ((size_t)(warp * kMats + m) * 16 + g) * kQTok + 8 * j + 2 * c;
                pp[0] = acc[m][j][0];
                pp[1] = acc[m][j][1];
                pp[8 * kQTok] = acc[m][j][2];
                pp[8 * kQTok + 1] = acc[m][j][3];
            }
        __syncthreads();
        // the warps' partials in fixed order, the row scale and the epilogue: thread (row, token)
        for (int q = threadIdx.x; q < 16 * kQTok; q += blockDim.x) {
            const int row = q / kQTok, tok = q % kQTok, o = r0 + row;
            if (tok >= nt) continue;
            float v[kMats];
#pragma unroll
            for (int m = 0; m < kMats; ++m) {
                float sm = 0.0f;
                for (int w = 0; w < kQWarps; ++w) sm += part[((size_t)(w * kMats + m) * 16 + row) * kQTok + tok];
                v[m] = sm * bf16f((m ? a.W1 : a.W0).scales[o]);
            }
            const int64_t i = (int64_t)(t0 + tok) * out + o;
            if constexpr (kMode == kQLinear) {
                a.yf[i] = v[0];
            } else if constexpr (kMode == kQGateUp) {
                a.yf[i] = silu(v[0]) * v[kMats - 1];
            } else {
                a.yb[i] = f2bf16(v[0] + (a.res ? bf16f(a.res[i]) : 0.0f));
            }
        }
    }
}

size_t mma_smem(int mode, int n) {
    const int planes = mode == kQDown ? 2 : 1, mats = mode == kQGateUp ? 2 : 1;
    return (size_t)planes * kQTok * (n + 8) * 2 + (size_t)kQWarps * mats * 16 * kQTok * 4;
}

// The tensor-core path applies: enough tokens, K a multiple of 64 per warp, whole 16-row
// tiles, 16-byte aligned packed rows and inputs, and the staging fits in shared memory.
bool mma_ok(int mode, const moe_mixed_tensor& W, const void* in, int T) {
    if (T < kQMinTokens || W.in % (64 * kQWarps) || W.out % 16) return false;
    if (((uintptr_t)W.packed & 15) || ((uintptr_t)in & 15)) return false;
    return mma_smem(mode, W.in) <= 220 * 1024;
}

template <int kMode>
cudaError_t launch_mma(const QArgs& a, cudaStream_t s) {
    static int cached = 0;
    const size_t smem = mma_smem(kMode, a.W0.in);
    cudaError_t e = ensure_smem((const void*)mixed_mma_kernel<kMode>, smem, cached);
    if (e != cudaSuccess) return e;
    mixed_mma_kernel<kMode><<<a.W0.out / 16, kQWarps * 32, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

#define MOEQ_MIXED_DISPATCH(MTV, CALL) \
    switch (MTV) {                       \
        case 1: CALL(1); break;          \
        case 2: CALL(2); break;          \
        case 4: CALL(4); break;          \
        default: CALL(8); break;         \
    }

cudaError_t launch_mixed_linear(const moe_mixed_tensor& W, int G, const uint16_t* x, int T, float* y, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    if (mma_ok(kQLinear, W, x, T)) {
        QArgs a = {};
        a.W0 = W;
        a.G = G;
        a.T = T;
        a.xb = x;
        a.yf = y;
        return launch_mma<kQLinear>(a, s);
    }
    const int mt = mt_for(T);
    const size_t smem = stage_bytes(W.in, mt);
    cudaError_t e = cudaSuccess;
#define MOEQ_CALL(M)                                                                                                 \
    {                                                                                                                \
        e = ensure_smem((const void*)mixed_linear_kernel<M>, smem, cache_lin[M]);                                     \
        if (e == cudaSuccess)                                                                                        \
            mixed_linear_kernel<M><<<(W.out + kMWarps - 1) / kMWarps, kMWarps * 32, smem, s>>>(W, G, x, T, y);       \
    }
    static int cache_lin[kMT + 1] = {0};
    MOEQ_MIXED_DISPATCH(mt, MOEQ_CALL)
#undef MOEQ_CALL
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_mixed_gate_up(const moe_mixed_tensor& g, const moe_mixed_tensor& u, int G, const uint16_t* x,
                                 int T, float* h, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    if (mma_ok(kQGateUp, g, x, T) && ((uintptr_t)u.packed & 15) == 0) {
        QArgs a = {};
        a.W0 = g;
        a.W1 = u;
        a.G = G;
        a.T = T;
        a.xb = x;
        a.yf = h;
        return launch_mma<kQGateUp>(a, s);
    }
    const int mt = mt_for(T);
    const size_t smem = stage_bytes(g.in, mt);
    cudaError_t e = cudaSuccess;
#define MOEQ_CALL(M)                                                                                                 \
    {                                                                                                                \
        e = ensure_smem((const void*)mixed_gate_up_kernel<M>, smem, cache_gu[M]);                                     \
        if (e == cudaSuccess)                                                                                        \
            mixed_gate_up_kernel<M><<<(g.out + kMWarps - 1) / kMWarps, kMWarps * 32, smem, s>>>(g, u, G, x, T, h);   \
    }
    static int cache_gu[kMT + 1] = {0};
    MOEQ_MIXED_DISPATCH(mt, MOEQ_CALL)
#undef MOEQ_CALL
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_mixed_down(const moe_mixed_tensor& d, int G, const float* h, int T, const uint16_t* residual,
                              uint16_t* y, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    if (mma_ok(kQDown, d, h, T)) {
        QArgs a = {};
        a.W0 = d;
        a.G = G;
        a.T = T;
        a.xf = h;
        a.yb = y;
        a.res = residual;
        return launch_mma<kQDown>(a, s);
    }
    const int mt = mt_for(T);
    const size_t smem = stage_bytes(d.in, mt);
    cudaError_t e = cudaSuccess;
#define MOEQ_CALL(M)                                                                                                 \
    {                                                                                                                \
        e = ensure_smem((const void*)mixed_down_kernel<M>, smem, cache_dn[M]);                                        \
        if (e == cudaSuccess)                                                                                        \
            mixed_down_kernel<M><<<(d.out + kMWarps - 1) / kMWarps, kMWarps * 32, smem, s>>>(d, G, h, T, residual, y); \
    }
    static int cache_dn[kMT + 1] = {0};
    MOEQ_MIXED_DISPATCH(mt, MOEQ_CALL)
#undef MOEQ_CALL
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace moeq
