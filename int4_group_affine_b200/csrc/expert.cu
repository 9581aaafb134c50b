// expert.cu - a4/a5/a6 on CUDA cores: expert-grouped int4 GEMV kernels with the
// unmerged LoRA delta, fused SwiGLU, and the fixed-order combine.
//
// Work is grouped by expert (the index build's groups): every CTA takes a tile
// of weight rows of one expert, streams those rows from HBM once with 16-byte
// loads, unpacks nibbles in registers and applies them to every token routed to
// that expert (chunks of kTok tokens staged in shared memory).  The dot product
// uses the group-affine factorisation sum_j (s q_j + b) x_j = s sum_j q_j x_j +
// b sum_j x_j over each 32-element chunk, so a weight costs one integer-to-float
// step and one FMA per token.
#include "common.cuh"

namespace moeq {
namespace {

constexpr int kTok = 4;          // tokens per shared-memory chunk
constexpr int kGUWarps = 8;      // gate/up: warps per CTA
constexpr int kGUPairs = 2;      // gate/up: (gate row, up row) pairs per warp
constexpr int kGURows = kGUWarps * kGUPairs;
constexpr int kDWarps = 8;       // down: warps per CTA
constexpr int kDRows = 16;       // down: output rows per CTA

// Physical float index of logical element j inside a token row staged in
// shared memory: each 32-element chunk is rotated by 4 * (chunk % 8) floats so
// that lanes reading the same offset of consecutive chunks hit different banks.
__device__ __forceinline__ int swz(int j) {
    const int c = j >> 5;
    return (c << 5) | (((j & 31) + ((c & 7) << 2)) & 31);
}

__device__ __forceinline__ const moe_lora_proj* lora_proj(const LayerArgs& L, int a, bool shared, int which) {
    if (a < 0 || a >= L.n_adapters) return nullptr;
    const moe_lora_ptrs& p = L.lora[a];
    const moe_lora_proj* q = which == 0 ? (shared ? &p.s_gate : &p.gate)
                           : which == 1 ? (shared ? &p.s_up : &p.up)
                                        : (shared ? &p.s_down : &p.down);
    return (q->A && q->B) ? q : nullptr;
}

// Stage kTok rows of length n (bf16 or fp32 source) into swizzled fp32 shared
// memory plus 32-element chunk sums.
template <typename Src>
__device__ void stage_rows(float* xs, float* xsum, const Src* const* rows, int nt, int n) {
    for (int i = threadIdx.x; i < kTok * n; i += blockDim.x) {
        const int tt = i / n, j = i % n;
        float v = 0.0f;
        if (tt < nt) {
            if constexpr (sizeof(Src) == 2) v = bf16f(rows[tt][j]);
            else v = rows[tt][j];
        }
        xs[tt * n + swz(j)] = v;
    }
    __syncthreads();
    const int nc = n / 32;
    for (int i = threadIdx.x; i < kTok * nc; i += blockDim.x) {
        const int tt = i / nc, c = i % nc;
        float s = 0.0f;
        for (int f = 0; f < 32; ++f) s += xs[tt * n + (c << 5) + f];
        xsum[i] = s;
    }
    __syncthreads();
}

// acc[tt] += sum over the 32 elements of chunk c of (s q + b) x[tt].
__device__ __forceinline__ void chunk_dot(const uint4 q4, int c, float s, float b, const float* xs,
                                          const float* xsum, int n, float* acc) {
    const uint32_t qw[4] = {q4.x, q4.y, q4.z, q4.w};
    float qf[32];
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int f = 0; f < 8; ++f) qf[w * 8 + f] = u2f_small((qw[w] >> (4 * f)) & 15u);
    const int rot = (c & 7) << 2;
#pragma unroll
    for (int tt = 0; tt < kTok; ++tt) {
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
        acc[tt] = fmaf(s, a, fmaf(b, xsum[tt * (n / 32) + c], acc[tt]));
    }
}

// --------------------------------------------------------------- LoRA A
// Grid (J, ceil(ndots / 4)): each warp one dot product A[mat][d] . v, where v is
// the token's input row (phase 0, gate and up: 2r dots) or the job's SwiGLU
// activation (phase 1, down: r dots).
__global__ void lora_a_kernel(Work wk, const __grid_constant__ LayerArgs L, int phase, const uint16_t* __restrict__ x) {
    const int p = blockIdx.x;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int d = blockIdx.y * 4 + warp;
    const int r = L.rank;
    const int ndots = phase == 0 ? 2 * r : r;
    if (d >= ndots || p >= wk.J) return;
    const int4 job = wk.perm[p];
    const int t = job.x, a = job.z, e = job.w;
    const bool shared = e == wk.E;
    const int64_t mat = shared ? 0 : e;
    float* out = phase == 0 ? wk.tgu + (int64_t)p * 2 * r + d : wk.td + (int64_t)p * r + d;
    const moe_lora_proj* lp = lora_proj(L, a, shared, phase == 0 ? (d < r ? 0 : 1) : 2);
    if (!lp) {
        if (lane == 0) *out = 0.0f;
        return;
    }
    const int dd = phase == 0 ? d % r : d;
    float acc = 0.0f;
    if (phase == 0) {
        const int n = L.H;
        const uint4* ar = reinterpret_cast<const uint4*>(lp->A + (mat * r + dd) * n);
        const uint4* xr = reinterpret_cast<const uint4*>(x + (int64_t)t * n);
        for (int v = lane; v < n / 8; v += 32) {
            const uint4 av = ar[v], xv = xr[v];
            const uint32_t aw[4] = {av.x, av.y, av.z, av.w}, xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                acc = fmaf(__uint_as_float(aw[k] << 16), __uint_as_float(xw[k] << 16), acc);
                acc = fmaf(__uint_as_float(aw[k] & 0xFFFF0000u), __uint_as_float(xw[k] & 0xFFFF0000u), acc);
            }
        }
    } else {
        const int n = shared ? L.Is : L.I;
        const uint4* ar = reinterpret_cast<const uint4*>(lp->A + (mat * r + dd) * n);
        const float* hr = wk.h + (int64_t)p * wk.Imax;
        for (int v = lane; v < n / 8; v += 32) {
            const uint4 av = ar[v];
            const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                acc = fmaf(__uint_as_float(aw[k] << 16), hr[v * 8 + 2 * k], acc);
                acc = fmaf(__uint_as_float(aw[k] & 0xFFFF0000u), hr[v * 8 + 2 * k + 1], acc);
            }
        }
    }
    acc = warp_sum(acc);
    if (lane == 0) *out = acc;
}

// ------------------------------------------------------------ gate / up
// Items (active group, tile of kGURows intermediate rows), grid-strided.  A warp
// owns kGUPairs rows i and computes gate row i and up row i together, so
// h = SiLU(g) * u is formed in registers.
__global__ void __launch_bounds__(kGUWarps * 32)
gate_up_kernel(Work wk, const __grid_constant__ LayerArgs L, const uint16_t* __restrict__ x) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);  // [kTok][H] swizzled
    float* xsum = xs + kTok * L.H;                   // [kTok][H/32]
    __shared__ int4 jobs[kTok];
    const int H = L.H;
    const int ntiles = (wk.Imax + kGURows - 1) / kGURows;
    const int nitems = *wk.n_active * ntiles;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int r = L.rank;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
        const int e = wk.active[item / ntiles];
        const int tile = item % ntiles;
        const bool shared = e == wk.E;
        const int I = shared ? L.Is : L.I;
        if (tile * kGURows >= I) continue;  // uniform across the CTA
        const moe_qtensor& Wg = shared ? L.s_gate : L.gate;
        const moe_qtensor& Wu = shared ? L.s_up : L.up;
        const int64_t mat = shared ? 0 : e;
        const int p0 = wk.goff[e], p1 = wk.goff[e + 1];
        const int ng = H / Wg.group;
        const int words = H / 8;
        for (int pc = p0; pc < p1; pc += kTok) {
            const int nt = min(kTok, p1 - pc);
            __syncthreads();
            if (threadIdx.x < kTok) jobs[threadIdx.x] = threadIdx.x < nt ? wk.perm[pc + threadIdx.x] : make_int4(0, 0, -1, 0);
            __syncthreads();
            const uint16_t* rows[kTok];
#pragma unroll
            for (int tt = 0; tt < kTok; ++tt) rows[tt] = x + (int64_t)jobs[tt].x * H;
            stage_rows(xs, xsum, rows, nt, H);
            for (int pr = 0; pr < kGUPairs; ++pr) {
                const int i = tile * kGURows + warp * kGUPairs + pr;
                if (i >= I) break;
                const int64_t row = mat * Wg.out + i;
                const uint4* gq = reinterpret_cast<const uint4*>(Wg.packed + row * words);
                const uint4* uq = reinterpret_cast<const uint4*>(Wu.packed + row * words);
                const uint16_t* gs_ = Wg.scales + row * ng;
                const uint16_t* gb_ = Wg.biases + row * ng;
                const uint16_t* us_ = Wu.scales + row * ng;
                const uint16_t* ub_ = Wu.biases + row * ng;
                float ag[kTok], au[kTok];
#pragma unroll
                for (int tt = 0; tt < kTok; ++tt) ag[tt] = au[tt] = 0.0f;
                for (int c = lane; c < H / 32; c += 32) {
                    const uint4 g4 = gq[c], u4 = uq[c];
                    const int g = (c * 32) / Wg.group;
                    chunk_dot(g4, c, bf16f(gs_[g]), bf16f(gb_[g]), xs, xsum, H, ag);
                    chunk_dot(u4, c, bf16f(us_[g]), bf16f(ub_[g]), xs, xsum, H, au);
                }
#pragma unroll
                for (int tt = 0; tt < kTok; ++tt) {
                    ag[tt] = warp_sum(ag[tt]);
                    au[tt] = warp_sum(au[tt]);
                }
                for (int tt = 0; tt < nt; ++tt) {
                    const int p = pc + tt;
                    const int a = jobs[tt].z;
                    float dg = 0.0f, du = 0.0f;
                    const moe_lora_proj* lg = lora_proj(L, a, shared, 0);
                    const moe_lora_proj* lu = lora_proj(L, a, shared, 1);
                    if (lg && lane < r) dg = bf16f(lg->B[(mat * I + i) * r + lane]) * wk.tgu[(int64_t)p * 2 * r + lane];
                    if (lu && lane < r) du = bf16f(lu->B[(mat * I + i) * r + lane]) * wk.tgu[(int64_t)p * 2 * r + r + lane];
                    for (int kk = lane + 32; kk < r; kk += 32) {
                        if (lg) dg += bf16f(lg->B[(mat * I + i) * r + kk]) * wk.tgu[(int64_t)p * 2 * r + kk];
                        if (lu) du += bf16f(lu->B[(mat * I + i) * r + kk]) * wk.tgu[(int64_t)p * 2 * r + r + kk];
                    }
                    dg = warp_sum(dg);
                    du = warp_sum(du);
                    if (lane == 0) {
                        const float gv = ag[tt] + L.scale * dg;
                        const float uv = au[tt] + L.scale * du;
                        wk.h[(int64_t)p * wk.Imax + i] = silu(gv) * uv;
                    }
                }
            }
        }
    }
}

// ------------------------------------------------------------------ down
// Items (active group, tile of kDRows output rows).  Rows of the down matrix are
// I/8 words; a row is split over `lpr` lanes (16-byte loads), 32/lpr rows per
// warp step.  Writes ypart[p][o] = w_p * (W_d h_p + scale * B_d t_d).
__global__ void __launch_bounds__(kDWarps * 32) down_kernel(Work wk, const __grid_constant__ LayerArgs L) {
    extern __shared__ float4 smem_f4[];
    float* hs = reinterpret_cast<float*>(smem_f4);  // [kTok][Imax] swizzled
    float* hsum = hs + kTok * wk.Imax;               // [kTok][Imax/32]
    __shared__ int4 jobs[kTok];
    __shared__ float wts[kTok];
    const int H = L.H;
    const int ntiles = (H + kDRows - 1) / kDRows;
    const int nitems = *wk.n_active * ntiles;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int r = L.rank;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
        const int e = wk.active[item / ntiles];
        const int tile = item % ntiles;
        const bool shared = e == wk.E;
        if (shared && wk.Is == 0) continue;  // no shared expert: combine skips these jobs
        const int I = shared ? L.Is : L.I;
        const moe_qtensor& Wd = shared ? L.s_down : L.down;
        const int64_t mat = shared ? 0 : e;
        const int p0 = wk.goff[e], p1 = wk.goff[e + 1];
        const int ng = I / Wd.group;
        const int nvec = I / 32;                       // 16-byte vectors per row
        int lpr = 1;                                   // lanes per row: largest power of two <= min(32, nvec)
        while (lpr * 2 <= min(32, nvec)) lpr *= 2;
        const int rpw = 32 / lpr;                      // rows per warp step
        const int sub = lane / lpr, sl = lane % lpr;
        for (int pc = p0; pc < p1; pc += kTok) {
            const int nt = min(kTok, p1 - pc);
            __syncthreads();
            if (threadIdx.x < kTok) {
                jobs[threadIdx.x] = threadIdx.x < nt ? wk.perm[pc + threadIdx.x] : make_int4(0, 0, -1, 0);
                wts[threadIdx.x] = threadIdx.x < nt ? wk.wperm[pc + threadIdx.x] : 0.0f;
            }
            __syncthreads();
            const float* rows[kTok];
#pragma unroll
            for (int tt = 0; tt < kTok; ++tt) rows[tt] = wk.h + (int64_t)(pc + (tt < nt ? tt : 0)) * wk.Imax;
            stage_rows(hs, hsum, rows, nt, I);
            for (int r0 = warp * rpw; r0 < kDRows; r0 += kDWarps * rpw) {
                const int o = tile * kDRows + r0 + sub;
                const bool live = o < H && (r0 + sub) < kDRows;
                float acc[kTok];
#pragma unroll
                for (int tt = 0; tt < kTok; ++tt) acc[tt] = 0.0f;
                if (live) {
                    const int64_t row = mat * Wd.out + o;
                    const uint4* dq = reinterpret_cast<const uint4*>(Wd.packed + row * (I / 8));
                    for (int c = sl; c < nvec; c += lpr) {
                        const int g = (c * 32) / Wd.group;
                        chunk_dot(dq[c], c, bf16f(Wd.scales[row * ng + g]), bf16f(Wd.biases[row * ng + g]), hs,
                                  hsum, I, acc);
                    }
                }
#pragma unroll
                for (int tt = 0; tt < kTok; ++tt)
                    for (int off = lpr / 2; off > 0; off >>= 1) acc[tt] += __shfl_xor_sync(0xffffffffu, acc[tt], off);
                for (int tt = 0; tt < nt; ++tt) {
                    const int p = pc + tt;
                    const moe_lora_proj* ld = lora_proj(L, jobs[tt].z, shared, 2);
                    float dd = 0.0f;
                    if (live && ld)
                        for (int kk = sl; kk < r; kk += lpr)
                            dd += bf16f(ld->B[(mat * H + o) * r + kk]) * wk.td[(int64_t)p * r + kk];
                    for (int off = lpr / 2; off > 0; off >>= 1) dd += __shfl_xor_sync(0xffffffffu, dd, off);
                    if (live && sl == 0) wk.ypart[(int64_t)p * H + o] = wts[tt] * (acc[tt] + L.scale * dd);
                }
            }
        }
    }
}

// --------------------------------------------------------------- combine
// y[t][o] = sum_{k<K} ypart[inv(t,k)][o] + ypart[inv(t,K)][o] (+ residual), in that order.
// Any alignment of y: one output per thread.
__global__ void combine_scalar_kernel(Work wk, const uint16_t* __restrict__ residual, uint16_t* __restrict__ y) {
    const int t = blockIdx.y;
    const int o = blockIdx.x * blockDim.x + threadIdx.x;
    if (o >= wk.H || t >= wk.T) return;
    float acc = 0.0f;
    const int kend = wk.K + (wk.Is > 0 ? 1 : 0);
    for (int k = 0; k < kend; ++k) acc += wk.ypart[(int64_t)wk.inv[(int64_t)t * (wk.K + 1) + k] * wk.H + o];
    if (residual) acc += bf16f(residual[(int64_t)t * wk.H + o]);
    y[(int64_t)t * wk.H + o] = f2bf16(acc);
}

__device__ __forceinline__ void combine4(const Work& wk, const uint16_t* __restrict__ residual,
                                         uint16_t* __restrict__ y, int t, int o4) {
    const int kend = wk.K + (wk.Is > 0 ? 1 : 0);
    float4 v[MOEQ_MAX_TOPK + 1];
#pragma unroll
    for (int k = 0; k <= MOEQ_MAX_TOPK; ++k) {
        v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (k < kend) {
            const int64_t row = wk.inv[(int64_t)t * (wk.K + 1) + k];
            v[k] = reinterpret_cast<const float4*>(wk.ypart + row * wk.H)[o4];
        }
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k <= MOEQ_MAX_TOPK; ++k) {
        if (k >= kend) break;
        acc.x += v[k].x;
        acc.y += v[k].y;
        acc.z += v[k].z;
        acc.w += v[k].w;
    }
    if (residual) {
        const uint2 r = reinterpret_cast<const uint2*>(residual + (int64_t)t * wk.H)[o4];
        acc.x += __uint_as_float(r.x << 16);
        acc.y += __uint_as_float(r.x & 0xFFFF0000u);
        acc.z += __uint_as_float(r.y << 16);
        acc.w += __uint_as_float(r.y & 0xFFFF0000u);
    }
    const uint2 out = make_uint2((uint32_t)f2bf16(acc.x) | ((uint32_t)f2bf16(acc.y) << 16),
                                 (uint32_t)f2bf16(acc.z) | ((uint32_t)f2bf16(acc.w) << 16));
    reinterpret_cast<uint2*>(y + (int64_t)t * wk.H)[o4] = out;
}

// The same for 8-byte aligned y and residual: a thread takes 4 consecutive outputs of one
// token, with the loads of all of the token's jobs in flight together.
__global__ void combine_kernel(Work wk, const uint16_t* __restrict__ residual, uint16_t* __restrict__ y) {
    const int t = blockIdx.y, o4 = blockIdx.x * blockDim.x + threadIdx.x;
    if (o4 * 4 < wk.H && t < wk.T) combine4(wk, residual, y, t, o4);
}


}  // namespace

static int g_num_sms = 0;
static int num_sms() {
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (g_num_sms <= 0) g_num_sms = 148;
    }
    return g_num_sms;
}

cudaError_t launch_lora_a(const Work& wk, const LayerArgs& L, int phase, const uint16_t* x, cudaStream_t s) {
    if (wk.T == 0 || L.n_adapters == 0 || L.rank == 0) return cudaSuccess;
    const int ndots = phase == 0 ? 2 * L.rank : L.rank;
    dim3 grid(wk.J, (ndots + 3) / 4);
    lora_a_kernel<<<grid, 128, 0, s>>>(wk, L, phase, x);
    return cudaGetLastError();
}

cudaError_t launch_gate_up(const Work& wk, const LayerArgs& L, const uint16_t* x, int max_groups, cudaStream_t s) {
    if (wk.T == 0) return cudaSuccess;
    const int ntiles = (wk.Imax + kGURows - 1) / kGURows;
    const int64_t items = (int64_t)max_groups * ntiles;
    const int grid = (int)(items < num_sms() * 4 ? items : num_sms() * 4);
    const size_t smem = (size_t)kTok * L.H * sizeof(float) + (size_t)kTok * (L.H / 32) * sizeof(float);
    static int cached = 0;
    cudaError_t e = ensure_smem((const void*)gate_up_kernel, smem, cached);
    if (e != cudaSuccess) return e;
    gate_up_kernel<<<grid, kGUWarps * 32, smem, s>>>(wk, L, x);
    return cudaGetLastError();
}

cudaError_t launch_down(const Work& wk, const LayerArgs& L, int max_groups, cudaStream_t s) {
    if (wk.T == 0) return cudaSuccess;
    const int ntiles = (L.H + kDRows - 1) / kDRows;
    const int64_t items = (int64_t)max_groups * ntiles;
    const int grid = (int)(items < num_sms() * 8 ? items : num_sms() * 8);
    const size_t smem = (size_t)kTok * wk.Imax * sizeof(float) + (size_t)kTok * (wk.Imax / 32) * sizeof(float);
    static int cached = 0;
    cudaError_t e = ensure_smem((const void*)down_kernel, smem, cached);
    if (e != cudaSuccess) return e;
    down_kernel<<<grid, kDWarps * 32, smem, s>>>(wk, L);
    return cudaGetLastError();
}

cudaError_t launch_combine(const Work& wk, const uint16_t* residual, uint16_t* y, cudaStream_t s) {
    if (wk.T == 0) return cudaSuccess;
    if (((uintptr_t)y & 7) || ((uintptr_t)residual & 7) || wk.H % 4) {
        dim3 grid((wk.H + 255) / 256, wk.T);
        combine_scalar_kernel<<<grid, 256, 0, s>>>(wk, residual, y);
    } else {
        dim3 grid((wk.H / 4 + 127) / 128, wk.T);
        combine_kernel<<<grid, 128, 0, s>>>(wk, residual, y);
    }
    return cudaGetLastError();
}

}  // namespace moeq
