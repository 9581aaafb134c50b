// pack.cu - a0: group-affine and mixed ternary/4-bit quantise-and-pack, and the
// dequantise export.  Setup-time kernels: correctness (bit-exact fp64 decisions)
// matters here, not speed.
#include "common.cuh"

namespace moeq {
namespace {

// bf16 is fp32 with the low half dropped (truncation toward zero).  Directed
// rounding of a double: first to fp32 in the same direction (exact intrinsics),
// then bump the truncated pattern by one unit when truncation went the wrong way.
__device__ uint16_t bf16_directed(double v, int dir) {
    float f = dir < 0 ? __double2float_rd(v) : __double2float_ru(v);
    uint32_t u = __float_as_uint(f);
    uint16_t t = (uint16_t)(u >> 16);
    if ((u & 0xFFFFu) == 0) return t;
    bool neg = (u >> 31) != 0;
    if (dir < 0) return neg ? (uint16_t)(t + 1) : t;
    return neg ? t : (uint16_t)(t + 1);
}

__device__ uint16_t bf16_nearest_even(double v) {
    uint16_t lo = bf16_directed(v, -1), hi = bf16_directed(v, +1);
    if (lo == hi) return lo;
    double dl = v - (double)bf16f(lo), dh = (double)bf16f(hi) - v;
    if (dl < dh) return lo;
    if (dh < dl) return hi;
    return (lo & 1u) ? hi : lo;
}

// One thread per (row, group).  b = group min rounded down, s = range/qmax
// rounded up, q = clamp(rint((w - b)/s)): every decision in fp64.
__global__ void pack_affine_kernel(const float* __restrict__ W, int64_t rows, int in, int group, int bits,
                                   uint32_t* __restrict__ packed, uint16_t* __restrict__ scales,
                                   uint16_t* __restrict__ biases) {
    const int ngroups = in / group;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= rows * ngroups) return;
    const int64_t r = gid / ngroups;
    const int g = (int)(gid % ngroups);
    const float* w = W + r * in + (int64_t)g * group;
    float lo = w[0], hi = w[0];
    for (int j = 1; j < group; ++j) {
        float v = w[j];
        lo = fminf(lo, v);
        hi = fmaxf(hi, v);
    }
    if (lo == 0.0f) lo = 0.0f;  // a minimum of -0 and +0 stores the bias +0
    const int qmax = (1 << bits) - 1;
    const uint16_t b16 = bf16_directed((double)lo, -1);
    const double b = (double)bf16f(b16);
    const double d = (double)hi - b;
    uint16_t s16 = 0;
    double s = 0.0;
    if (d > 0.0) {
        s16 = bf16_directed(d / (double)qmax, +1);
        s = (double)bf16f(s16);
    }
    scales[gid] = s16;
    biases[gid] = b16;
    const int per_word = 32 / bits;
    uint32_t* out = packed + (r * in + (int64_t)g * group) / per_word;
    for (int wd = 0; wd < group / per_word; ++wd) {
        uint32_t word = 0;
        for (int f = 0; f < per_word; ++f) {
            uint32_t q = 0;
            if (s > 0.0) {
                double t = rint(((double)w[wd * per_word + f] - b) / s);
                t = fmin(fmax(t, 0.0), (double)qmax);
                q = (uint32_t)t;
            }
            word |= q << (f * bits);
        }
        out[wd] = word;
    }
}

// One thread per output row of a mixed matrix.
__global__ void pack_mixed_kernel(const float* __restrict__ W, int out, int in, int G,
                                  uint32_t* __restrict__ packed, uint16_t* __restrict__ scales) {
    const int o = blockIdx.x * blockDim.x + threadIdx.x;
    if (o >= out) return;
    const float* w = W + (int64_t)o * in;
    uint32_t* pw = packed + mixed_row_offset(o, in, G);
    const double eps = 1e-5;
    if (G > 0 && o % G == 0) {
        double m = 0.0;
        for (int j = 0; j < in; ++j) m = fmax(m, fabs((double)w[j]));
        const uint16_t s16 = bf16_nearest_even(fmax(m / 7.0, eps));
        scales[o] = s16;
        const double s = (double)bf16f(s16);
        for (int wd = 0; wd < in / 8; ++wd) {
            uint32_t word = 0;
            for (int f = 0; f < 8; ++f) {
                double t = fmin(fmax(rint((double)w[wd * 8 + f] / s), -7.0), 7.0);
                word |= (uint32_t)((int)t + 8) << (4 * f);
            }
            pw[wd] = word;
        }
    } else {
        double sum = 0.0;
        for (int j = 0; j < in; ++j) sum += fabs((double)w[j]);
        const uint16_t s16 = bf16_nearest_even(fmax(2.0 * (sum / (double)in), eps));
        scales[o] = s16;
        const double s = (double)bf16f(s16);
        for (int wd = 0; wd < in / 16; ++wd) {
            uint32_t word = 0;
            for (int f = 0; f < 16; ++f) {
                double t = fmin(fmax(rint((double)w[wd * 16 + f] / s), -1.0), 1.0);
                word |= (uint32_t)((int)t + 1) << (2 * f);
            }
            pw[wd] = word;
        }
    }
}

__global__ void dequant_affine_kernel(moe_qtensor t, float* __restrict__ out) {
    const int64_t total = (int64_t)t.n * t.out * t.in;
    const int per_word = 32 / t.bits;
    const uint32_t mask = (1u << t.bits) - 1u;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = i / t.in;
        const int j = (int)(i % t.in);
        const uint32_t word = t.packed[(row * t.in + j) / per_word];
        const uint32_t q = (word >> ((j % per_word) * t.bits)) & mask;
        const int64_t gi = row * (t.in / t.group) + j / t.group;
        out[i] = __fmaf_rn(bf16f(t.scales[gi]), u2f_small(q), bf16f(t.biases[gi]));
    }
}

__global__ void dequant_mixed_kernel(moe_mixed_tensor t, int G, float* __restrict__ out) {
    const int64_t total = (int64_t)t.out * t.in;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int o = (int)(i / t.in);
        const int j = (int)(i % t.in);
        const uint32_t* pw = t.packed + mixed_row_offset(o, t.in, G);
        int q;
        if (G > 0 && o % G == 0) q = (int)((pw[j / 8] >> (4 * (j % 8))) & 15u) - 8;
        else q = (int)((pw[j / 16] >> (2 * (j % 16))) & 3u) - 1;
        out[i] = bf16f(t.scales[o]) * (float)q;
    }
}

}  // namespace

cudaError_t launch_pack_affine(const float* W, int64_t rows, int in, int group, int bits, uint32_t* packed,
                               uint16_t* scales, uint16_t* biases, cudaStream_t s) {
    const int64_t n = rows * (in / group);
    if (n == 0) return cudaSuccess;
    const int threads = 128;
    pack_affine_kernel<<<(unsigned)((n + threads - 1) / threads), threads, 0, s>>>(W, rows, in, group, bits, packed,
                                                                                 scales, biases);
    return cudaGetLastError();
}

cudaError_t launch_pack_mixed(const float* W, int out, int in, int G, uint32_t* packed, uint16_t* scales,
                              cudaStream_t s) {
    if (out == 0) return cudaSuccess;
    pack_mixed_kernel<<<(out + 63) / 64, 64, 0, s>>>(W, out, in, G, packed, scales);
    return cudaGetLastError();
}

cudaError_t launch_dequant_affine(const moe_qtensor& t, float* out, cudaStream_t s) {
    const int64_t total = (int64_t)t.n * t.out * t.in;
    if (total == 0) return cudaSuccess;
    const int64_t blocks = (total + 255) / 256;
    dequant_affine_kernel<<<(unsigned)(blocks < 148 * 32 ? blocks : 148 * 32), 256, 0, s>>>(t, out);
    return cudaGetLastError();
}

cudaError_t launch_dequant_mixed(const moe_mixed_tensor& t, int G, float* out, cudaStream_t s) {
    const int64_t total = (int64_t)t.out * t.in;
    if (total == 0) return cudaSuccess;
    const int64_t blocks = (total + 255) / 256;
    dequant_mixed_kernel<<<(unsigned)(blocks < 148 * 32 ? blocks : 148 * 32), 256, 0, s>>>(t, G, out);
    return cudaGetLastError();
}

}  // namespace moeq
