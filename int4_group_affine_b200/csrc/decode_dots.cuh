// decode_dots.cuh - device pieces shared by the fused decode kernels: bounded
// waits on bulk copies, bulk-copy windows, staging of activation rows into
// swizzled fp32 shared memory, and the int4 / int8 / bf16 row dot products
// that read them.
#pragma once

#include "tc.cuh"

namespace moeq {
namespace {

constexpr int kDecThreads = 512;  // threads per CTA of the fused decode kernels

// Wait (bounded) for phase 0 of a bulk-copy mbarrier; gives up at once if *abort is set.
__device__ bool copies_landed(uint64_t* bar, int32_t* status, volatile int* abort, uint64_t limit_ns) {
    if (tc::mbar_try_wait(bar, 0)) return true;
    const uint64_t t0 = tc::globaltimer_ns();
    for (;;) {
        if (tc::mbar_try_wait(bar, 0)) return true;
        if (*abort) return false;
        if (tc::globaltimer_ns() - t0 > limit_ns) {
            raise_status(status, MOE_ERR_TIMEOUT);
            *abort = 1;
            return false;
        }
    }
}

// Bulk copy of the 16-byte-aligned window around [src, src + bytes) to dst (16-byte
// aligned shared memory), completing on `bar`; returns where src's first byte lands and
// adds the window's size to *tx.  The host checks that every window stays inside its
// tensor (16-byte aligned base, size a multiple of 16).
__device__ __forceinline__ const unsigned char* win_load(unsigned char* dst, const void* src, uint32_t bytes,
                                                         uint64_t* bar, uint32_t* tx) {
    const uintptr_t s = (uintptr_t)src, a0 = s & ~(uintptr_t)15, a1 = (s + bytes + 15) & ~(uintptr_t)15;
    if (bytes) {
        const uint32_t span = (uint32_t)(a1 - a0);
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                         tc::smem_u32(dst)),
                     "l"(a0), "r"(span), "r"(tc::smem_u32(bar))
                     : "memory");
        *tx += span;
    }
    return dst + (s - a0);
}
__device__ __forceinline__ uint32_t win_span(const void* src, uint32_t bytes) {
    const uintptr_t s = (uintptr_t)src;
    return bytes ? (uint32_t)(((s + bytes + 15) & ~(uintptr_t)15) - (s & ~(uintptr_t)15)) : 0u;
}


// Stage nv bf16 rows of length n (n % 32 == 0) into swizzled fp32 shared memory
// with 32-element chunk sums; each thread has four 16-byte loads in flight.  With
// `scale`, each value becomes bf16(x * scale[v]) (the normalised block input).
__device__ void stage_bf16(float* dst, float* dsum, const uint16_t* src, int nv, int n, const float* scale) {
    const int per = n / 8, total = nv * per;
    const int lim = (total + 31) / 32 * 32;
    for (int i0 = threadIdx.x; i0 < lim; i0 += 4 * kDecThreads) {
        uint4 raw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * kDecThreads;
            raw[j] = make_uint4(0u, 0u, 0u, 0u);
            if (i < total) raw[j] = reinterpret_cast<const uint4*>(src + (int64_t)(i / per) * n)[i % per];
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * kDecThreads;
            if (i >= lim) break;  // uniform across the warp
            const bool live = i < total;
            const int v = live ? i / per : 0, q = live ? i % per : 0;
            float f[8];
            const uint32_t w[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                f[2 * k] = __uint_as_float(w[k] << 16);
                f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
            }
            if (scale && live)
#pragma unroll
                for (int k = 0; k < 8; ++k) f[k] = bf16f(f2bf16(f[k] * scale[v]));
            const int c = q / 4, o = (q % 4) * 8, rot = (c & 7) << 2;
            float s = 0.0f;
#pragma unroll
            for (int k = 0; k < 8; ++k) s += f[k];
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            if (live) {
                float* d = dst + v * n + (c << 5);
                *reinterpret_cast<float4*>(d + ((o + rot) & 31)) = make_float4(f[0], f[1], f[2], f[3]);
                *reinterpret_cast<float4*>(d + ((o + 4 + rot) & 31)) = make_float4(f[4], f[5], f[6], f[7]);
                if ((q % 4) == 0) dsum[v * (n / 32) + c] = s;
            }
        }
    }
}

// Same for fp32 rows written by other CTAs (read from L2), row stride `ld`, by the
// threads [t0, t0 + nthr) (whole warps); each thread has four loads in flight.
__device__ void stage_f32(float* dst, float* dsum, const float* src, int ld, int nv, int n, int t0, int nthr) {
    const int per = n / 4, total = nv * per;
    const int lim = (total + 31) / 32 * 32;
    for (int i0 = threadIdx.x - t0; i0 < lim; i0 += 4 * nthr) {
        float4 f[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * nthr;
            f[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < total) f[j] = __ldcg(reinterpret_cast<const float4*>(src + (int64_t)(i / per) * ld) + i % per);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * nthr;
            if (i >= lim) break;  // uniform across the warp (lim and nthr are multiples of 32)
            const bool live = i < total;
            const int v = live ? i / per : 0, q = live ? i % per : 0;
            const int c = q / 8, o = (q % 8) * 4, rot = (c & 7) << 2;
            float s = f[j].x + f[j].y + f[j].z + f[j].w;
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            if (live) {
                *reinterpret_cast<float4*>(dst + v * n + (c << 5) + ((o + rot) & 31)) = f[j];
                if ((q % 8) == 0) dsum[v * (n / 32) + c] = s;
            }
        }
    }
}

// 32 nibbles q -> 32 floats 128 + q: the nibble goes into bits 16..19 of 128.0f (whose
// upper 7 mantissa bits count in units of 1), one shift and one and-or each.  Products
// (128 + q) x are exact in fp32 for bf16 x; the caller removes the 128 through the bias
// term: s sum (128 + q) x + (b - 128 s) sum x = sum (s q + b) x.
__device__ __forceinline__ void unpack4(const uint4 q4, float* qf) {
    const uint32_t qw[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int f = 0; f < 8; ++f) {
            const uint32_t at16 = f <= 4 ? qw[w] << (16 - 4 * f) : qw[w] >> (4 * f - 16);
            qf[w * 8 + f] = __uint_as_float((at16 & 0x000F0000u) | 0x43000000u);
        }
}

// sum over chunk c of q[j] * v[j] for a staged (swizzled) vector row v.
__device__ __forceinline__ float chunk_qdot(const float* qf, const float* vrow, int c) {
    const float* vr = vrow + (c << 5);
    const int rot = (c & 7) << 2;
    float a = 0.0f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const float4 xv = *reinterpret_cast<const float4*>(vr + ((4 * u + rot) & 31));
        a = fmaf(qf[4 * u + 0], xv.x, a);
        a = fmaf(qf[4 * u + 1], xv.y, a);
        a = fmaf(qf[4 * u + 2], xv.z, a);
        a = fmaf(qf[4 * u + 3], xv.w, a);
    }
    return a;
}

// acc[m] += sum_j (s q_j + b) v_m[j] over one int4 row of length n (<= 4096), for
// staged vectors v_m = vbase + vid[m] * n (m < nv <= MT), by a group of `lpt`
// lanes (sl = lane index in the group).  All of the row's loads are issued
// before any use.
// (Not inlined: one copy of the code serves every call site, which keeps the
// kernel's instruction footprint small; each launch runs every phase once.)
template <int MT>
__device__ __noinline__ void dot_int4(const uint32_t* __restrict__ prow, const uint16_t* __restrict__ srow,
                                         const uint16_t* __restrict__ brow, int group, int n, const float* vbase,
                                         const float* vsum, const int* vid, int nv, float* acc, int sl, int lpt) {
    constexpr int kIt = 4;
    const uint4* p4 = reinterpret_cast<const uint4*>(prow);
    const int nc = n / 32;
    uint4 q[kIt];
    float s[kIt], b[kIt];
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = sl + lpt * it;
        if (c < nc) {
            q[it] = p4[c];
            const int g = (c * 32) / group;
            s[it] = bf16f(srow[g]);
            b[it] = bf16f(brow[g]);
        }
    }
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = sl + lpt * it;
        if (c >= nc) break;
        float qf[32];
        unpack4(q[it], qf);
        const float b128 = fmaf(-128.0f, s[it], b[it]);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m >= nv) break;
            const float a = chunk_qdot(qf, vbase + vid[m] * n, c);
            acc[m] = fmaf(s[it], a, fmaf(b128, vsum[vid[m] * nc + c], acc[m]));
        }
    }
}

// Same for an int8 row (H <= 4096), full warp, vectors v_m = vbase + m * n.
template <int MT>
__device__ __noinline__ void dot_int8(const uint32_t* __restrict__ prow, const uint16_t* __restrict__ srow,
                                         const uint16_t* __restrict__ brow, int group, int n, const float* vbase,
                                         const float* vsum, int nv, float* acc, int lane) {
    constexpr int kIt = 4;
    const uint4* p4 = reinterpret_cast<const uint4*>(prow);
    const int nc = n / 32;
    uint4 q0[kIt], q1[kIt];
    float s[kIt], b[kIt];
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = lane + 32 * it;
        if (c < nc) {
            q0[it] = p4[2 * c];
            q1[it] = p4[2 * c + 1];
            const int g = (c * 32) / group;
            s[it] = bf16f(srow[g]);
            b[it] = bf16f(brow[g]);
        }
    }
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = lane + 32 * it;
        if (c >= nc) break;
        const uint32_t qw[8] = {q0[it].x, q0[it].y, q0[it].z, q0[it].w, q1[it].x, q1[it].y, q1[it].z, q1[it].w};
        float qf[32];
#pragma unroll
        for (int w = 0; w < 8; ++w)
#pragma unroll
            for (int f = 0; f < 4; ++f) qf[w * 4 + f] = u2f_small((qw[w] >> (8 * f)) & 255u);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m >= nv) break;
            const float a = chunk_qdot(qf, vbase + m * n, c);
            acc[m] = fmaf(s[it], a, fmaf(b[it], vsum[m * nc + c], acc[m]));
        }
    }
}

// sum_j A[j] v[j] for a bf16 row A of length n (<= 4096) and one staged vector
// (lane partial; the caller reduces).  All loads first.
__device__ __noinline__ float dot_bf16(const uint16_t* __restrict__ arow, int n, const float* v, int lane) {
    constexpr int kIt = 4;
    const uint4* a4 = reinterpret_cast<const uint4*>(arow);
    const int nc = n / 32;
    uint4 q[kIt][4];
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = lane + 32 * it;
        if (c < nc)
#pragma unroll
            for (int u = 0; u < 4; ++u) q[it][u] = a4[4 * c + u];
    }
    float acc = 0.0f;
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = lane + 32 * it;
        if (c >= nc) break;
        const int rot = (c & 7) << 2;
        const float* vr = v + (c << 5);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint32_t aw[4] = {q[it][u].x, q[it][u].y, q[it][u].z, q[it][u].w};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float4 xv = *reinterpret_cast<const float4*>(vr + ((8 * u + 4 * h + rot) & 31));
                acc = fmaf(__uint_as_float(aw[2 * h] << 16), xv.x, acc);
                acc = fmaf(__uint_as_float(aw[2 * h] & 0xFFFF0000u), xv.y, acc);
                acc = fmaf(__uint_as_float(aw[2 * h + 1] << 16), xv.z, acc);
                acc = fmaf(__uint_as_float(aw[2 * h + 1] & 0xFFFF0000u), xv.w, acc);
            }
        }
    }
    return acc;
}

__device__ __forceinline__ float group_sum(float v, int lpt) {
    for (int o = lpt / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ const moe_lora_proj* dlora(const LayerArgs& L, int a, bool shared, int which) {
    if (a < 0 || a >= L.n_adapters) return nullptr;
    const moe_lora_ptrs& p = L.lora[a];
    const moe_lora_proj* q = which == 0 ? (shared ? &p.s_gate : &p.gate)
                           : which == 1 ? (shared ? &p.s_up : &p.up)
                                        : (shared ? &p.s_down : &p.down);
    return (q->A && q->B) ? q : nullptr;
}


// Order-preserving map of a float (NaN taken as -inf) onto unsigned integers, and back.
__device__ __forceinline__ uint32_t okey(float z) {
    const uint32_t u = z != z ? 0xff800000u : __float_as_uint(z);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float okey_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

}  // namespace
}  // namespace moeq
