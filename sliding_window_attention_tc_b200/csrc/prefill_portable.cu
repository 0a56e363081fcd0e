// Portable prefill of the Tensor Cache layer: float32 SIMT arithmetic for any
// supported shape (1 <= d_k, d_v <= 128, any W and C, float32 or bf16
// inputs).  It is the float32 path, and the path for shapes the tensor-core
// kernel does not take.
//
// "Tensor Cache: Eviction-conditioned Associative Memory for Transformers":
//  - L1 (§3.1, eq. (1)): softmax over keys t-W+1..t, scaled by 1/sqrt(d_k);
//  - L2 (§3.2, Fig. 2 step (3); abstract and §1 for the chunk scan): the
//    evictions e = 0..E-1 (E = max(0, T-W), token e leaves the window at
//    step e+W) are cut into chunks of C.  A chunk-state kernel runs the
//    weighted-sum scan  S_{c+1} = lambda^{C_c} S_c + eta sum_i lambda^{C_c-1-i}
//    k_i v_i^T  per head and stores every chunk's starting state S_c;
//  - the read at step t (eviction e = t-W, chunk c = e / C, offset r) is
//    m_t = lambda^{r+1} q_t S_c + eta sum_{i=cC}^{e} lambda^{e-i} <q_t,k_i> v_i
//    (inter-chunk read of the stored state plus the decay-weighted
//    intra-chunk part), which is q_t A_t with A_t including token t-W;
//  - fusion (Fig. 2 step (5)): y_t = y_local_t + sigmoid(g) m_t.

#include "tc_internal.cuh"

namespace tc {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxD = 128;
constexpr int kMaxPerThread = kMaxD * kMaxD / kThreads;  // 64

__host__ __device__ inline int64_t evictions(int64_t T, int64_t W) { return T > W ? T - W : 0; }
__host__ __device__ inline int64_t num_chunks(int64_t E, int64_t C) { return (E + C - 1) / C; }

// Row tau of the combined halo + new sequence of one (b,h): halo rows first.
template <typename T>
__device__ __forceinline__ const T *kv_row(const void *halo, const void *base, int64_t bh,
                                           int64_t n_halo, int64_t T_new, int d, int64_t tau) {
    return tau < n_halo ? reinterpret_cast<const T *>(halo) + (bh * n_halo + tau) * d
                        : reinterpret_cast<const T *>(base) + (bh * T_new + (tau - n_halo)) * d;
}

// Chunk scan over one head's evictions; stores S_c (state at the start of
// chunk c) for c = 0..nC-1 and A_final = the state after all evictions.
template <typename T>
__global__ void __launch_bounds__(kThreads) chunk_state_kernel(PrefillParams p, float *states,
                                                               int64_t nC) {
    constexpr int KT = 32;
    __shared__ float sk[KT][kMaxD + 1], sv[KT][kMaxD + 1];
    __shared__ float sw[KT];
    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x;
    const int h = (int)(bh % p.H);
    const int dk = p.dk, dv = p.dv, nel = dk * dv;
    const int64_t E = evictions(p.T + p.n_halo, p.W), C = p.C;
    const double lam = p.lam[h], eta = p.eta[h];

    // thread -> column col, rows row0 + i * rstep
    const int rstep = kThreads / dv;
    const int col = tid % dv, row0 = tid / dv;
    const bool active = tid < rstep * dv;
    float S[kMaxPerThread], D[kMaxPerThread];
#pragma unroll
    for (int i = 0; i < kMaxPerThread; ++i) {
        const int r = row0 + i * rstep;
        S[i] = (p.A_init && active && r < dk) ? p.A_init[bh * nel + r * dv + col] : 0.f;
    }

    for (int64_t c = 0; c < nC; ++c) {
        float *Sc = states + (bh * nC + c) * nel;
        if (active) {
#pragma unroll
            for (int i = 0; i < kMaxPerThread; ++i) {
                const int r = row0 + i * rstep;
                if (r < dk) Sc[r * dv + col] = S[i];
            }
        }
        const int64_t c0 = c * C;
        const int64_t Cc = (E - c0 < C) ? E - c0 : C;
#pragma unroll
        for (int i = 0; i < kMaxPerThread; ++i) D[i] = 0.f;
        float Vs = 0.f;  // chunk-mean ablation: sum of the chunk's values in column col
        for (int64_t i0 = 0; i0 < Cc; i0 += KT) {
            const int nt = (int)((Cc - i0 < KT) ? Cc - i0 : KT);
            __syncthreads();
            for (int x = tid; x < nt * dk; x += kThreads)
                sk[x / dk][x % dk] = to_f32(
                    kv_row<T>(p.halo_k, p.k, bh, p.n_halo, p.T, dk, c0 + i0 + x / dk)[x % dk]);
            for (int x = tid; x < nt * dv; x += kThreads)
                sv[x / dv][x % dv] = to_f32(
                    kv_row<T>(p.halo_v, p.v, bh, p.n_halo, p.T, dv, c0 + i0 + x / dv)[x % dv]);
            if (tid < nt)
                sw[tid] = p.chunk_mean ? 1.0f
                                       : (float)(eta * pow(lam, (double)(Cc - 1 - (i0 + tid))));
            __syncthreads();
            if (p.chunk_mean && active) {
                // ablation: sums of the chunk's keys and values (their means below)
                for (int j = 0; j < nt; ++j) {
#pragma unroll
                    for (int i = 0; i < kMaxPerThread; ++i) {
                        const int r = row0 + i * rstep;
                        if (r < dk) D[i] += sk[j][r];
                    }
                    Vs += sv[j][col];
                }
            } else if (active) {
                for (int j = 0; j < nt; ++j) {
                    const float wv = sw[j] * sv[j][col];
#pragma unroll
                    for (int i = 0; i < kMaxPerThread; ++i) {
                        const int r = row0 + i * rstep;
                        if (r < dk) D[i] = fmaf(sk[j][r], wv, D[i]);
                    }
                }
            }
        }
        if (p.chunk_mean) {
            // the chunk-mean shortcut: A <- lam A + eta kbar vbar^T once per chunk
            const float w = (float)(eta / ((double)Cc * (double)Cc)) * Vs;
#pragma unroll
            for (int i = 0; i < kMaxPerThread; ++i) S[i] = fmaf((float)lam, S[i], w * D[i]);
        } else {
            const float dec = (float)pow(lam, (double)Cc);
#pragma unroll
            for (int i = 0; i < kMaxPerThread; ++i) S[i] = fmaf(dec, S[i], D[i]);
        }
    }
    if (p.A_final && active) {
        float *A = p.A_final + bh * nel;
#pragma unroll
        for (int i = 0; i < kMaxPerThread; ++i) {
            const int r = row0 + i * rstep;
            if (r < dk) A[r * dv + col] = S[i];
        }
    }
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// One warp per query row, ROWS consecutive rows per CTA sharing key tiles.
// mrow: with the delta-rule write, m_t of every new row from
// delta_l2_kernel (the L2 read is then taken from there, not from chunk
// states); null for the outer-product write.
template <typename Tin>
__global__ void __launch_bounds__(kThreads) prefill_rows_kernel(PrefillParams p,
                                                                const float *states, int64_t nC,
                                                                const float *mrow) {
    constexpr int ROWS = kThreads / 32, KT = 32, CPL = kMaxD / 32;
    __shared__ float sk[KT][kMaxD + 1], sv[KT][kMaxD + 1];
    __shared__ float sq[ROWS][kMaxD];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.y;
    const int h = (int)(bh % p.H);
    const int dk = p.dk, dv = p.dv;
    // rows of q and y are the new tokens; positions t below are in the
    // combined halo + new sequence (t = row + n_halo)
    const int64_t T_new = p.T, nh = p.n_halo, T = T_new + nh, W = p.W, C = p.C;
    const int64_t t0 = nh + (int64_t)blockIdx.x * ROWS;
    const int64_t t = t0 + warp;
    const bool row_ok = t < T;
    const bool use_l2 = !p.l1_only;
    const Tin *qb = reinterpret_cast<const Tin *>(p.q) + bh * T_new * dk;

    for (int x = tid; x < ROWS * dk; x += kThreads) {
        const int64_t tt = t0 + x / dk;
        sq[x / dk][x % dk] = tt < T ? to_f32(qb[(tt - nh) * dk + x % dk]) : 0.f;
    }

    const float lam = p.lam[h], eta = p.eta[h];
    const float log2lam = (float)log2((double)lam);
    const float scale = (float)(1.4426950408889634 / sqrt((double)dk));
    const int64_t win_lo = t - W + 1 > 0 ? t - W + 1 : 0;
    const int64_t e = t - W;                       // eviction read at step t
    const bool has_l2 = use_l2 && row_ok && e >= 0 && !mrow;
    const int64_t ch = has_l2 ? e / C : 0;
    const int64_t intra_lo = ch * C;

    // key range needed by the CTA's rows
    const int64_t t_last = (t0 + ROWS - 1 < T - 1) ? t0 + ROWS - 1 : T - 1;
    int64_t lo = t0 - W + 1 > 0 ? t0 - W + 1 : 0;
    if (use_l2 && t_last >= W) {
        const int64_t e_first = t0 - W > 0 ? t0 - W : 0;
        const int64_t l2lo = (e_first / C) * C;
        if (l2lo < lo) lo = l2lo;
    }

    float acc[CPL], macc[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) acc[i] = macc[i] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;

    for (int64_t j0 = lo; j0 <= t_last; j0 += KT) {
        const int nt = (int)((t_last - j0 + 1 < KT) ? t_last - j0 + 1 : KT);
        __syncthreads();
        for (int x = tid; x < nt * dk; x += kThreads)
            sk[x / dk][x % dk] = to_f32(kv_row<Tin>(p.halo_k, p.k, bh, nh, T_new, dk, j0 + x / dk)[x % dk]);
        for (int x = tid; x < nt * dv; x += kThreads)
            sv[x / dv][x % dv] = to_f32(kv_row<Tin>(p.halo_v, p.v, bh, nh, T_new, dv, j0 + x / dv)[x % dv]);
        __syncthreads();
        if (!row_ok) continue;
        const int64_t j = j0 + lane;
        const bool in_win = lane < nt && j >= win_lo && j <= t;
        const bool in_intra = has_l2 && lane < nt && j >= intra_lo && j <= e;
        float dot = 0.f;
        if (in_win || in_intra)
            for (int r = 0; r < dk; ++r) dot = fmaf(sq[warp][r], sk[lane][r], dot);
        const float s = in_win ? dot * scale : -INFINITY;
        const float w = in_intra ? eta * exp2f((float)(e - j) * log2lam) * dot : 0.f;
        const float m_new = fmaxf(m_run, warp_max(s));
        float pj = 0.f;
        if (m_new != -INFINITY) {
            const float corr = exp2f(m_run - m_new);
            pj = exp2f(s - m_new);
            l_run = l_run * corr + warp_sum(pj);
#pragma unroll
            for (int i = 0; i < CPL; ++i) acc[i] *= corr;
            m_run = m_new;
        }
        for (int jj = 0; jj < nt; ++jj) {
            const float pb = __shfl_sync(0xffffffffu, pj, jj);
            const float wb = __shfl_sync(0xffffffffu, w, jj);
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int c = lane + 32 * i;
                if (c < dv) {
                    const float vv = sv[jj][c];
                    acc[i] = fmaf(pb, vv, acc[i]);
                    macc[i] = fmaf(wb, vv, macc[i]);
                }
            }
        }
    }
    if (!row_ok) return;

    float gate = 0.f;
    if (mrow && use_l2 && e >= 0) {
        gate = sigmoidf_acc(p.g[h]);
        const float *mr = mrow + (bh * T_new + (t - nh)) * dv;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            if (c < dv) macc[i] = mr[c];
        }
    }
    if (has_l2) {
        // inter-chunk read: lambda^{r+1} q_t S_c
        gate = sigmoidf_acc(p.g[h]);
        const int64_t r = e - intra_lo;
        const float dec = (float)exp2((double)(r + 1) * (double)log2((double)lam));
        const float *S = states + (bh * nC + ch) * dk * dv;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            if (c < dv) {
                float mi = 0.f;
                for (int rr = 0; rr < dk; ++rr) mi = fmaf(sq[warp][rr], S[rr * dv + c], mi);
                macc[i] = fmaf(dec, mi, macc[i]);
            }
        }
    }
    Tin *y = reinterpret_cast<Tin *>(p.y) + (bh * T_new + (t - nh)) * dv;
    const float inv_l = 1.0f / l_run;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const int c = lane + 32 * i;
        if (c < dv) y[c] = from_f32<Tin>(acc[i] * inv_l + gate * macc[i]);
    }
}

// Delta-rule write (Fig. 2 step (3) with update = k_old (v_old - k_old^T A)^T):
// each write reads A, so the writes of one (b,h) run in token order here.  A
// lives in shared memory; for every new row t with an eviction behind it the
// kernel records m_t = q_t A_t in mrow, and it leaves A_final.
template <typename T>
__global__ void __launch_bounds__(kThreads) delta_l2_kernel(PrefillParams p, float *mrow) {
    extern __shared__ float sA[];  // [dk][dv]
    __shared__ float sk[kMaxD], sv[kMaxD], sq[kMaxD], su[kMaxD];
    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x;
    const int h = (int)(bh % p.H);
    const int dk = p.dk, dv = p.dv, nel = dk * dv;
    const int64_t nh = p.n_halo, T_new = p.T, T_all = nh + T_new, W = p.W;
    const float lam = p.lam[h], eta = p.eta[h];
    for (int x = tid; x < nel; x += kThreads) sA[x] = p.A_init ? p.A_init[bh * nel + x] : 0.f;
    const T *qb = reinterpret_cast<const T *>(p.q) + bh * T_new * dk;
    // tokens before max(W, n_halo) neither evict nor have a query to answer
    for (int64_t tau = (W > nh ? W : nh) < T_all ? (W > nh ? W : nh) : T_all; tau < T_all; ++tau) {
        const bool evict = tau >= W;
        const bool query = !p.state_only;
        __syncthreads();
        if (evict) {
            for (int x = tid; x < dk; x += kThreads)
                sk[x] = to_f32(kv_row<T>(p.halo_k, p.k, bh, nh, T_new, dk, tau - W)[x]);
            for (int x = tid; x < dv; x += kThreads)
                sv[x] = to_f32(kv_row<T>(p.halo_v, p.v, bh, nh, T_new, dv, tau - W)[x]);
        }
        if (query)
            for (int x = tid; x < dk; x += kThreads) sq[x] = to_f32(qb[(tau - nh) * dk + x]);
        __syncthreads();
        if (evict) {
            for (int c = tid; c < dv; c += kThreads) {
                float pred = 0.f;
                for (int r = 0; r < dk; ++r) pred = fmaf(sk[r], sA[r * dv + c], pred);
                su[c] = sv[c] - pred;
            }
            __syncthreads();
            for (int x = tid; x < nel; x += kThreads)
                sA[x] = fmaf(lam, sA[x], eta * sk[x / dv] * su[x % dv]);
            __syncthreads();
        }
        if (query) {
            for (int c = tid; c < dv; c += kThreads) {
                float m = 0.f;
                for (int r = 0; r < dk; ++r) m = fmaf(sq[r], sA[r * dv + c], m);
                mrow[(bh * T_new + (tau - nh)) * dv + c] = m;
            }
        }
    }
    __syncthreads();
    if (p.A_final)
        for (int x = tid; x < nel; x += kThreads) p.A_final[bh * nel + x] = sA[x];
}

template <typename T>
cudaError_t launch_t(const PrefillParams &p, cudaStream_t s) {
    const int64_t BH = p.B * p.H;
    if (BH == 0) return cudaSuccess;
    if (p.delta_rule && !p.l1_only && p.n_halo == 0) {
        // chunked delta-rule memory, then the window part reads m from mrow
        cudaError_t e = launch_delta_chunked(p, std::is_same<T, float>::value ? TC_F32 : TC_BF16, false, s);
        if (e != cudaSuccess) return e;
        if (p.T > 0 && !p.state_only) {
            const dim3 grid((unsigned)((p.T + 7) / 8), (unsigned)BH);
            prefill_rows_kernel<T><<<grid, kThreads, 0, s>>>(p, nullptr, 0,
                                                             reinterpret_cast<const float *>(p.workspace));
        }
        return cudaGetLastError();
    }
    if (p.delta_rule && !p.l1_only) {
        // a continued sequence (halo): the writes in token order
        float *mrow = reinterpret_cast<float *>(p.workspace);
        const size_t smem = (size_t)p.dk * p.dv * sizeof(float);
        cudaError_t e = cudaFuncSetAttribute(delta_l2_kernel<T>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        delta_l2_kernel<T><<<(unsigned)BH, kThreads, smem, s>>>(p, mrow);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        if (p.T > 0 && !p.state_only) {
            const dim3 grid((unsigned)((p.T + 7) / 8), (unsigned)BH);
            prefill_rows_kernel<T><<<grid, kThreads, 0, s>>>(p, nullptr, 0, mrow);
        }
        return cudaGetLastError();
    }
    const int64_t nC = p.l1_only ? 0 : num_chunks(evictions(p.T + p.n_halo, p.W), p.C);
    float *states = reinterpret_cast<float *>(p.workspace);
    if (!p.l1_only) {
        chunk_state_kernel<T><<<(unsigned)BH, kThreads, 0, s>>>(p, states, nC);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (p.T > 0 && !p.state_only) {
        const dim3 grid((unsigned)((p.T + 7) / 8), (unsigned)BH);
        prefill_rows_kernel<T><<<grid, kThreads, 0, s>>>(p, states, nC, nullptr);
    }
    return cudaGetLastError();
}

}  // namespace

size_t portable_workspace_bytes(const tc_prefill_desc &d, int64_t n_halo) {
    if (d.flags & TC_PREFILL_L1_ONLY) return 0;
    if (d.flags & TC_PREFILL_DELTA_RULE) {
        if (n_halo == 0) return delta_chunked_workspace_bytes(d);  // m_t rows and the chunk buffers
        // token order: m_t of every new row
        return (d.flags & TC_PREFILL_STATE_ONLY) ? 0 : (size_t)(d.B * d.H * d.T * d.dv) * sizeof(float);
    }
    const int64_t nC = num_chunks(evictions(d.T + n_halo, d.W), d.C);
    return (size_t)(d.B * d.H * nC * d.dk * d.dv) * sizeof(float);
}

cudaError_t launch_prefill_portable(const PrefillParams &p, tc_dtype dtype, cudaStream_t s) {
    return dtype == TC_BF16 ? launch_t<__nv_bfloat16>(p, s) : launch_t<float>(p, s);
}

}  // namespace tc
