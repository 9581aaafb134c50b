// decode_cdots.cuh - device pieces of the decode kernels that hand values between
// CTAs through epoch-tagged words (the chain and cluster decode kernels): publishing
// and polling the words, staging activation rows, compact row dots and the warp top-K.
#pragma once

#include "decode_dots.cuh"

namespace moeq {
namespace {

constexpr int kCW = 16;  // warps per CTA
constexpr int kCT = kCW * 32;
static_assert(kCT == kDecThreads, "one block size for the staging helpers");
constexpr int kGB = 8;   // words one thread polls per pass

// ------------------------------------------------------------ tagged words
__device__ __forceinline__ void publish(uint64_t* p, float v, uint32_t tag) {
    const unsigned long long w = ((unsigned long long)tag << 32) | __float_as_uint(v);
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ unsigned long long peek(const uint64_t* p) {
    unsigned long long w;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
    return w;
}
__device__ __forceinline__ bool fresh(unsigned long long w, uint32_t tag) { return (uint32_t)(w >> 32) == tag; }
__device__ __forceinline__ float wval(unsigned long long w) { return __uint_as_float((uint32_t)w); }

// Poll one word until it carries `tag` (bounded: MOE_ERR_TIMEOUT and *abort after
// limit_ns; gives up at once when *abort is already set).  Returns its value or 0.
__device__ __noinline__ float spin(const uint64_t* p, uint32_t tag, int32_t* status, volatile int* abort,
                                   uint64_t limit_ns) {
    const uint64_t t0 = tc::globaltimer_ns();
    for (uint32_t i = 0;; ++i) {
        const unsigned long long w = peek(p);
        if (fresh(w, tag)) return wval(w);
        if ((i & 7) == 7) {
            if (*abort) return 0.0f;
            if (tc::globaltimer_ns() - t0 > limit_ns) {
                raise_status(status, MOE_ERR_TIMEOUT);
                *abort = 1;
                return 0.0f;
            }
        }
        __nanosleep(32);  // leave the issue slots to the warps that compute
    }
}

__device__ __forceinline__ unsigned long long ld_acq64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// One thread: wait (bounded, with a short back-off between polls) until *p >= target
// (ge) or *p == target; acquire semantics.  False on timeout (MOE_ERR_TIMEOUT, *abort).
__device__ __noinline__ bool wait_word(const unsigned long long* p, unsigned long long target, bool ge,
                                       int32_t* status, volatile int* abort, uint64_t limit_ns) {
    const uint64_t t0 = tc::globaltimer_ns();
    for (uint32_t i = 0;; ++i) {
        const unsigned long long v = ld_acq64(p);
        if (ge ? v >= target : v == target) return true;
        if (*abort) return false;
        if ((i & 7) == 7 && tc::globaltimer_ns() - t0 > limit_ns) {
            raise_status(status, MOE_ERR_TIMEOUT);
            *abort = 1;
            return false;
        }
        __nanosleep(64);
    }
}

// Every thread of the CTA: dst[i] = value of word src[i] for i < n, all of a thread's
// loads of a pass in flight together.
__device__ void gather_range(const uint64_t* src, int n, float* dst, uint32_t tag, int32_t* status,
                             volatile int* abort, uint64_t limit_ns) {
    for (int base = 0; base < n; base += kGB * kCT) {
        unsigned long long w[kGB];
#pragma unroll
        for (int b = 0; b < kGB; ++b) {
            const int i = base + b * kCT + (int)threadIdx.x;
            w[b] = i < n ? peek(src + i) : 0ull;
        }
#pragma unroll
        for (int b = 0; b < kGB; ++b) {
            const int i = base + b * kCT + (int)threadIdx.x;
            if (i < n) dst[i] = fresh(w[b], tag) ? wval(w[b]) : spin(src + i, tag, status, abort, limit_ns);
        }
    }
}

// Position of element i of a staged (swizzled) row: 32-element chunks, 4-float groups
// rotated by the chunk index (the layout stage_bf16 / stage_f32 write).
__device__ __forceinline__ int swz(int i) {
    const int c = i >> 5, p = i & 31;
    return (c << 5) + (((p & ~3) + ((c & 7) << 2)) & 31) + (p & 3);
}

// Compact row dots for the chain kernel.  A launch runs most of its code once, so the
// time of a step is set by the instructions it has to fetch, not by those it executes:
// these loop over 32-element chunks with one chunk's body unrolled, instead of unrolling
// several chunks.
//
// acc[m] += sum_j (s q_j + b) v_m[j] over one int4 row of length n, staged vectors
// v_m = vbase + vid[m] * n, by lpt lanes (sl = lane in the group).  The nibble q goes
// into the mantissa of 128.0f; the 128 is taken back through the bias term
// (s sum (128 + q) v + (b - 128 s) sum v).
template <int MT>
__device__ __noinline__ void cdot_int4(const uint32_t* __restrict__ prow, const uint16_t* __restrict__ srow,
                                       const uint16_t* __restrict__ brow, int group, int n, const float* vbase,
                                       const float* vsum, const int* vid, int nv, float* acc, int sl, int lpt) {
    const uint4* p4 = reinterpret_cast<const uint4*>(prow);
    const int nc = n / 32, gsh = 31 - __clz(group >> 5);  // (group: a power of two, 32 or more)
#pragma unroll 1
    for (int c = sl; c < nc; c += lpt) {
        const int g = c >> gsh;
        const float s = bf16f(srow[g]), b128 = fmaf(-128.0f, s, bf16f(brow[g]));
        const uint4 q4 = p4[c];
        const uint32_t qw[4] = {q4.x, q4.y, q4.z, q4.w};
        const int rot = (c & 7) << 2;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m >= nv) break;
            const float* vr = vbase + vid[m] * n + (c << 5);
            float a = 0.0f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float4 x0 = *reinterpret_cast<const float4*>(vr + ((8 * w + rot) & 31));
                const float4 x1 = *reinterpret_cast<const float4*>(vr + ((8 * w + 4 + rot) & 31));
                const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                for (int f = 0; f < 8; ++f) {
                    const uint32_t at16 = f <= 4 ? qw[w] << (16 - 4 * f) : qw[w] >> (4 * f - 16);
                    a = fmaf(__uint_as_float((at16 & 0x000F0000u) | 0x43000000u), xv[f], a);
                }
            }
            acc[m] = fmaf(s, a, fmaf(b128, vsum[vid[m] * nc + c], acc[m]));
        }
    }
}

// The same for an int8 row, full warp, vectors v_m = vbase + m * n.
template <int MT>
__device__ __noinline__ void cdot_int8(const uint32_t* __restrict__ prow, const uint16_t* __restrict__ srow,
                                       const uint16_t* __restrict__ brow, int group, int n, const float* vbase,
                                       const float* vsum, int nv, float* acc, int lane) {
    const uint4* p4 = reinterpret_cast<const uint4*>(prow);
    const int nc = n / 32, gsh = 31 - __clz(group >> 5);  // (group: a power of two, 32 or more)
#pragma unroll 1
    for (int c = lane; c < nc; c += 32) {
        const int g = c >> gsh;
        const float s = bf16f(srow[g]), b = bf16f(brow[g]);
        const int rot = (c & 7) << 2;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m >= nv) break;
            const float* vr = vbase + m * n + (c << 5);
            float a = 0.0f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 q4 = p4[2 * c + h];
                const uint32_t qw[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const float4 xv = *reinterpret_cast<const float4*>(vr + ((16 * h + 4 * w + rot) & 31));
                    a = fmaf(u2f_small(qw[w] & 255u), xv.x, a);
                    a = fmaf(u2f_small((qw[w] >> 8) & 255u), xv.y, a);
                    a = fmaf(u2f_small((qw[w] >> 16) & 255u), xv.z, a);
                    a = fmaf(u2f_small(qw[w] >> 24), xv.w, a);
                }
            }
            acc[m] = fmaf(s, a, fmaf(b, vsum[m * nc + c], acc[m]));
        }
    }
}

// bf16 rows (n elements, 16-byte aligned) into the swizzled fp32 layout with 32-element
// chunk sums, optionally scaled (the normalised block input); a thread takes 8 elements.
__device__ void cstage_bf16(float* dst, float* dsum, const uint16_t* src, int nv, int n, const float* scale) {
    const int per = n / 8, total = nv * per, lim = (total + 31) / 32 * 32;
#pragma unroll 1
    for (int i = threadIdx.x; i < lim; i += kCT) {
        const bool live = i < total;
        const int v = live ? i / per : 0, q = live ? i % per : 0;
        const uint4 raw = live ? reinterpret_cast<const uint4*>(src + (int64_t)v * n)[q] : make_uint4(0, 0, 0, 0);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        float f[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            f[2 * k] = __uint_as_float(w[k] << 16);
            f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
        }
        if (scale && live)
#pragma unroll
            for (int k = 0; k < 8; ++k) f[k] = bf16f(f2bf16(f[k] * scale[v]));
        float sum = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) sum += f[k];
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        if (live) {
            const int c = q / 4, o = (q % 4) * 8, rot = (c & 7) << 2;
            float* d = dst + v * n + (c << 5);
            *reinterpret_cast<float4*>(d + ((o + rot) & 31)) = make_float4(f[0], f[1], f[2], f[3]);
            *reinterpret_cast<float4*>(d + ((o + 4 + rot) & 31)) = make_float4(f[4], f[5], f[6], f[7]);
            if ((q % 4) == 0) dsum[v * (n / 32) + c] = sum;
        }
    }
}

// sum_j A[j] v[j] for a bf16 row A of length n already in shared memory and one staged
// vector (lane partial; the caller reduces): lane takes 32-element chunks lane, lane + 32, ...
__device__ __forceinline__ float sdot_bf16(const uint16_t* arow, int n, const float* v, int lane) {
    const uint4* a4 = reinterpret_cast<const uint4*>(arow);
    float acc = 0.0f;
    for (int c = lane; c < n / 32; c += 32) {
        const int rot = (c & 7) << 2;
        const float* vr = v + (c << 5);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint4 q = a4[4 * c + u];
            const uint32_t aw[4] = {q.x, q.y, q.z, q.w};
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

// Top-K of one token's logits z[0..E) by one warp, E <= 32 * kC: lane holds experts
// lane + 32 c; K rounds of a warp max on order-preserving keys, equal keys to the lower
// expert index; weights exp(z_k - z_max) renormalised over the K.
template <int kC>
__device__ __forceinline__ void warp_topk(const float* z, int E, int K, int lane, int* idx, float* w) {
    uint32_t kv[kC];
#pragma unroll
    for (int c = 0; c < kC; ++c) {
        const int e = lane + 32 * c;
        kv[c] = e < E ? okey(z[e]) : 0u;
    }
    uint32_t myk = 0u;
    int mye = 0;
    for (int k = 0; k < K; ++k) {
        uint32_t bk = 0u;
        int bc = -1;
#pragma unroll
        for (int c = 0; c < kC; ++c)
            if (kv[c] > bk) {
                bk = kv[c];
                bc = c;
            }
        const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
        const int me = (int)__reduce_min_sync(0xffffffffu, (bc >= 0 && bk == mk) ? (unsigned)(lane + 32 * bc)
                                                                                   : 0x7fffffffu);
        if ((me & 31) == lane) {
#pragma unroll
            for (int c = 0; c < kC; ++c)
                if (c == (me >> 5)) kv[c] = 0u;
        }
        if (lane == k) {
            myk = mk;
            mye = me < E ? me : 0;
        }
    }
    const float zk = myk ? okey_value(myk) : -INFINITY;
    const float z0 = __shfl_sync(0xffffffffu, zk, 0);
    const float ev = lane < K ? (z0 > -INFINITY ? expf(zk - z0) : 1.0f) : 0.0f;
    const float sum = warp_sum(ev);
    if (lane < K) {
        idx[lane] = mye;
        w[lane] = ev / sum;
    }
}

// Bulk-copy window issue helper: nothing for bytes == 0 or a null source.
__device__ __forceinline__ const unsigned char* win(unsigned char* dst, const void* src, uint32_t bytes,
                                                    uint64_t* bar, uint32_t* tx) {
    if (!src || !bytes) return nullptr;
    return win_load(dst, src, bytes, bar, tx);
}

// L2 policy for weight rows: evict first.  A decode call streams its weights through L2
// once, and they should not push out what every call reuses (the kernels' code, the
// tagged words, the activations).
__device__ __forceinline__ uint64_t l2_stream_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// win() for weight rows, with the L2 policy `pol`.
__device__ __forceinline__ const unsigned char* winp(uint64_t pol, unsigned char* dst, const void* src,
                                                     uint32_t bytes, uint64_t* bar, uint32_t* tx) {
    if (!src || !bytes) return nullptr;
    const uintptr_t s = (uintptr_t)src, a0 = s & ~(uintptr_t)15, a1 = (s + bytes + 15) & ~(uintptr_t)15;
    const uint32_t span = (uint32_t)(a1 - a0);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            tc::smem_u32(dst)),
        "l"(a0), "r"(span), "r"(tc::smem_u32(bar)), "l"(pol)
        : "memory");
    *tx += span;
    return dst + (s - a0);
}

__device__ __forceinline__ uint32_t warp_total(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace
}  // namespace moeq
