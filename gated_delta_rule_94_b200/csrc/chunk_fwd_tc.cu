// chunk_fwd_tc.cu -- chunkwise gated delta rule on the sm_100a tensor cores
// (bf16 operands, fp32 accumulation in TMEM, fp32 state), d_k = d_v = 128.
//
// The chunkwise algorithm of "Moonshot AI's New Attention Architecture: Key
// Innovations Explained" (sec. 3, state recurrence and causal output) with the
// UT/WY transform of "OSDN: Improving Delta Rule with Provable Online
// Preconditioning in Linear Attention" (sec. 2.1, chunk Gram matrix + WY),
// for a scalar (or no) forget gate.  Per chunk of C = 64 tokens, h the
// entering state M = S^T [d_k][d_v], G the in-chunk log-decay cumsum:
//   S  = [K; Q] K^T                 (one 128-row MMA: K K^T and Q K^T)
//   A  = StrictTril(beta_r e^(G_r-G_i) (K K^T)_ri),  P = Tril(e^(G_r-G_i) (Q K^T)_ri)
//   T  = (I + A)^-1                 (forward substitution, fp32 CUDA cores)
//   W^T = K^T (T diag(beta e^G))^T  (MN-major K tile, M = d_k = 128)
//   X  = [T diag(beta); 0] V        = [U; 0]
//   X += [-W; Q_bar] h              -> rows 0..63: D = U - W h, rows 64..127: Q_bar h
//   X += [0; P] D                   -> rows 64..127: O = Q_bar h + P D
//   h  = e^(G_C) h + K^T (diag(e^(G_C - G_i)) D)
// Every product is a tcgen05.mma with M = 128, operands in 128 B-swizzled
// shared memory: the K/Q/V tiles exactly as TMA loads them (K-major for the
// token rows, MN-major when tokens are the reduction dimension), the other
// operands written by the threads in the same canonical layouts.
//
// One CTA of 4 warps owns one (batch, head) and walks its chunks in order;
// thread t owns TMEM lane t.  TMA prefetches the next chunk's K/Q while the
// current one is processed.  Every mbarrier wait is bounded; a wait that gives
// up sets the library status word and the CTA leaves the loop.
#include "common.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int C = 64;
constexpr int D = 128;
constexpr int NT = 128;
constexpr int LDF = 68;  // fp32 row stride of the A / T scratch (16 B-aligned rows)

// Shared memory layout (bytes from a 1 KB-aligned base).
constexpr uint32_t KQ_STAGE = 32768;         // [K_b0 | Q_b0 | K_b1 | Q_b1], 8 KB each
constexpr uint32_t OFF_KQ = 0;               // 2 stages
constexpr uint32_t OFF_V = 65536;            // [V_b0 | V_b1], 8 KB each
constexpr uint32_t OFF_TW = 81920;           // T diag(beta e^G), K-major [64 r][64 i]
constexpr uint32_t OFF_TU = 90112;           // T diag(beta), followed by ...
constexpr uint32_t OFF_Z = 98304;            // ... an 8 KB zero block, followed by ...
constexpr uint32_t OFF_P = 106496;           // ... P, K-major [64 r][64 i]
constexpr uint32_t OFF_WQ = 114688;          // MN-major [d][64 r]: -W^T block, Q_bar^T block
constexpr uint32_t OFF_HB = 147456;          // h (bf16) MN-major [d][64 v] x 2 blocks; after
constexpr uint32_t OFF_DL = 147456;          //   the c-MMA: D  [i][64 v] x 2 blocks
constexpr uint32_t OFF_DT = 163840;          //   and D~ = diag(e^(G_C-G_i)) D
constexpr uint32_t OFF_AF = 180224;          // A fp32 [64][LDF]
constexpr uint32_t OFF_TF = OFF_AF + 64 * LDF * 4;
constexpr uint32_t OFF_SMALL = OFF_TF + 64 * LDF * 4;   // G, e^G, e^(G_C-G), beta
constexpr uint32_t OFF_BAR = OFF_SMALL + 4 * 64 * 4;
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;     // alignment slack
static_assert(OFF_TF + 64 * LDF * 4 == OFF_SMALL, "layout");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns (512 allocated).
constexpr uint32_t TM_H = 0;      // state, lanes d, 128 columns v (fp32)
constexpr uint32_t TM_X = 128;    // [U->D ; Q_bar h->O], lanes r / 64 + r, 128 columns v
constexpr uint32_t TM_S = 256;    // [K K^T ; Q K^T], 64 columns
constexpr uint32_t TM_W = 320;    // W^T, lanes d, 64 columns r

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&t);
}

__device__ __forceinline__ void st_row_chunk(uint8_t* tile, int row, int j, const float* v,
                                             float scale) {
    uint4 w;
    w.x = pack_bf16(v[0] * scale, v[1] * scale);
    w.y = pack_bf16(v[2] * scale, v[3] * scale);
    w.z = pack_bf16(v[4] * scale, v[5] * scale);
    w.w = pack_bf16(v[6] * scale, v[7] * scale);
    *reinterpret_cast<uint4*>(tile + sw128_offset(row, 8 * j)) = w;
}

// T = (I + A)^-1 for strictly lower-triangular A (64 x 64, fp32), blocked in
// 16 x 16 tiles: the four diagonal tiles by column-parallel substitution, then
// the off-diagonal tiles by distance, T_ij = -T_ii sum_{j<=k<i} A_ik T_kj.
// The strictly upper tiles of Tm serve as scratch for the inner sums.
__device__ __forceinline__ void forward_substitution(const float* A, float* Tm, int tid) {
    if (tid < 64) {
        const int o = 16 * (tid >> 4), c = tid & 15;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < r; ++i) acc = fmaf(A[(o + r) * LDF + o + i], x[i], acc);
            x[r] = (r == c) ? 1.f : (r < c ? 0.f : -acc);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tm[(o + r) * LDF + o + c] = x[r];
    }
    __syncthreads();
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
        const int nb = 4 - d;
        for (int e = tid; e < nb * 256; e += NT) {
            const int j = e >> 8, i = j + d, r = (e >> 4) & 15, c = e & 15;
            const float* arow = A + (16 * i + r) * LDF;
            float acc = 0.f;
#pragma unroll 1
            for (int k = j; k < i; ++k) {
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    acc = fmaf(arow[16 * k + q], Tm[(16 * k + q) * LDF + 16 * j + c], acc);
            }
            Tm[(16 * j + r) * LDF + 16 * i + c] = acc;
        }
        __syncthreads();
        for (int e = tid; e < nb * 256; e += NT) {
            const int j = e >> 8, i = j + d, r = (e >> 4) & 15, c = e & 15;
            float acc = 0.f;
#pragma unroll
            for (int q = 0; q < 16; ++q)
                if (q <= r)
                    acc = fmaf(Tm[(16 * i + r) * LDF + 16 * i + q], Tm[(16 * j + q) * LDF + 16 * i + c], acc);
            Tm[(16 * i + r) * LDF + 16 * j + c] = -acc;
        }
        __syncthreads();
    }
}

struct TcMaps {
    CUtensorMap q, k, v;
};

template <int GATE>
__global__ void __launch_bounds__(NT, 1)
chunk_fwd_tc_kernel(const __grid_constant__ TcMaps maps, const ChunkParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    float* sG = reinterpret_cast<float*>(sm + OFF_SMALL);
    float* sGam = sG + 64;
    float* sFt = sG + 128;
    float* sBeta = sG + 192;
    float* Af = reinterpret_cast<float*>(sm + OFF_AF);
    float* Tf = reinterpret_cast<float*>(sm + OFF_TF);
    uint64_t* bar_kq = reinterpret_cast<uint64_t*>(sm + OFF_BAR);   // [2]
    uint64_t* bar_v = bar_kq + 2;
    uint64_t* bar_mma = bar_kq + 3;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H, T = p.T;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int NC = (T + C - 1) / C;
    const __nv_bfloat16* gq = static_cast<const __nv_bfloat16*>(p.g);
    const __nv_bfloat16* gb = static_cast<const __nv_bfloat16*>(p.beta);
    int failed = 0;
    uint32_t mma_phase = 0;

    if (tid == 0) {
        mbar_init(&bar_kq[0], 1);
        mbar_init(&bar_kq[1], 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        s_abort = 0;
        prefetch_tmap(&maps.q);
        prefetch_tmap(&maps.k);
        prefetch_tmap(&maps.v);
    }
    if (warp == 0) {
        tmem_alloc(&s_tmem, 512);
        tmem_relinquish();
    }
    for (int i = tid; i < 512; i += NT) reinterpret_cast<uint4*>(sm + OFF_Z)[i] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tH = tmem + TM_H, tX = tmem + TM_X, tS = tmem + TM_S, tW = tmem + TM_W;

    auto load_kq = [&](int n, int s) {
        mbar_arrive_expect_tx(&bar_kq[s], 4 * 8192);
        uint8_t* st = sm + OFF_KQ + s * KQ_STAGE;
        for (int blk = 0; blk < 2; ++blk) {
            tma_load_3d(st + blk * 16384, &maps.k, &bar_kq[s], h * D + 64 * blk, n * C, b);
            tma_load_3d(st + blk * 16384 + 8192, &maps.q, &bar_kq[s], h * D + 64 * blk, n * C, b);
        }
    };
    auto load_v = [&](int n) {
        mbar_arrive_expect_tx(bar_v, 2 * 8192);
        for (int blk = 0; blk < 2; ++blk)
            tma_load_3d(sm + OFF_V + blk * 8192, &maps.v, bar_v, h * D + 64 * blk, n * C, b);
    };
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
        if (!mbar_wait(bar, parity, &failed)) {
            atomicOr(p.status, kStatusTimeout);
            s_abort = 1;
        }
        __syncwarp();
    };

    // initial state -> TMEM, row d = tid
    {
        const float* s0 = p.s0 ? p.s0 + ((size_t)bh * D + tid) * D : nullptr;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 16) {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = s0 ? s0[c0 + j] : 0.f;
            tmem_st16(tH + lane_off + c0, v);
        }
        tmem_wait_st();
    }
    if (tid == 0 && NC > 0) {
        load_kq(0, 0);
        load_v(0);
    }
    float g_next = 0.f, b_next = 0.f;
    if (tid < 64 && tid < T) {
        const size_t tok = ((size_t)b * T + tid) * H + h;
        b_next = __bfloat162float(gb[tok]);
        if constexpr (GATE == kGateScalar) g_next = __bfloat162float(gq[tok]);
    }

#pragma unroll 1
    for (int n = 0; n < NC; ++n) {
        const int s = n & 1;
        const int t0 = n * C;
        const int nval = min(C, T - t0);
        uint8_t* stage = sm + OFF_KQ + s * KQ_STAGE;
        const uint32_t stage_a = sb + OFF_KQ + s * KQ_STAGE;

        // ---- gates of this chunk
        if (tid < 64) {
            sG[tid] = g_next;
            sBeta[tid] = b_next;
        }
        __syncthreads();
        if (warp == 0) {
            if constexpr (GATE == kGateScalar) {
                const float a0 = sG[2 * lane], a1 = sG[2 * lane + 1];
                float incl = a0 + a1;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += y;
                }
                float excl = __shfl_up_sync(0xffffffffu, incl, 1);
                if (lane == 0) excl = 0.f;
                const float G0 = excl + a0, G1 = incl;
                const float Gl = __shfl_sync(0xffffffffu, incl, 31);
                sG[2 * lane] = G0;
                sG[2 * lane + 1] = G1;
                sGam[2 * lane] = expf(G0);
                sGam[2 * lane + 1] = expf(G1);
                sFt[2 * lane] = expf(Gl - G0);
                sFt[2 * lane + 1] = expf(Gl - G1);
            } else {
                sG[2 * lane] = sG[2 * lane + 1] = 0.f;
                sGam[2 * lane] = sGam[2 * lane + 1] = 1.f;
                sFt[2 * lane] = sFt[2 * lane + 1] = 1.f;
            }
        }
        // ---- S = [K; Q] K^T
        if (tid == 0) {
            if (mbar_wait(&bar_kq[s], (n >> 1) & 1, &failed)) {
                const uint32_t id = idesc_bf16_f32(128, 64, false, false);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t a = stage_a + (k >> 2) * 16384 + (k & 3) * 32;
                    mma_bf16(tS, sdesc_sw128(a, 16, 1024), sdesc_sw128(a, 16, 1024), id, k > 0);
                }
            }
            mma_commit(bar_mma);
            if (n + 1 < NC) {
                fence_async_smem();
                load_kq(n + 1, s ^ 1);
            }
        }
        if (tid < 64 && n + 1 < NC) {
            g_next = 0.f;
            b_next = 0.f;
            if (t0 + C + tid < T) {
                const size_t tok = ((size_t)b * T + t0 + C + tid) * H + h;
                b_next = __bfloat162float(gb[tok]);
                if constexpr (GATE == kGateScalar) g_next = __bfloat162float(gq[tok]);
            }
        }
        wait_all(&bar_kq[s], (n >> 1) & 1);
        __syncthreads();
        if (s_abort) break;

        // ---- Q_bar^T (MN-major [d][64 r]) = e^(G_r) Q[r][d], thread d
        {
            const int d = tid, dc = d & 63;
            const uint8_t* qt = stage + (d >> 6) * 16384 + 8192;
            uint8_t* dst = sm + OFF_WQ + 16384;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint32_t w[4];
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    const int r0 = 8 * j + 2 * q2;
                    const float x0 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(qt + sw128_offset(r0, dc)));
                    const float x1 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(qt + sw128_offset(r0 + 1, dc)));
                    w[q2] = pack_bf16(x0 * sGam[r0], x1 * sGam[r0 + 1]);
                }
                *reinterpret_cast<uint4*>(dst + sw128_offset(d, 8 * j)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        // ---- A (fp32) and P (bf16) from S
        wait_all(bar_mma, mma_phase & 1);
        ++mma_phase;
        tc_fence_after();
        {
            float sv[64];
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_ld16(tS + lane_off + 16 * j, *reinterpret_cast<float(*)[16]>(sv + 16 * j));
            tmem_wait_ld();
            reg_fence(sv);
            if (tid < 64) {
                const int r = tid;
                const float Gr = sG[r], br = sBeta[r];
                float* arow = Af + r * LDF;
#pragma unroll
                for (int i = 0; i < 64; ++i) arow[i] = (i < r) ? br * expf(Gr - sG[i]) * sv[i] : 0.f;
            } else {
                const int r = tid - 64;
                const float Gr = sG[r];
#pragma unroll
                for (int i = 0; i < 64; ++i) sv[i] = (i <= r) ? expf(Gr - sG[i]) * sv[i] : 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) st_row_chunk(sm + OFF_P, r, j, sv + 8 * j, 1.f);
            }
        }
        fence_async_smem();
        __syncthreads();
        if (s_abort) break;

        // ---- T = (I + A)^-1, then T diag(beta e^G) and T diag(beta) as bf16
        forward_substitution(Af, Tf, tid);
        {
            const int r = tid >> 1, half = tid & 1;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int j = 4 * half + jj;
                float tw[8], tu[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int i = 8 * j + e;
                    const float tv = (i <= r) ? Tf[r * LDF + i] : 0.f;
                    tu[e] = tv * sBeta[i];
                    tw[e] = tu[e] * sGam[i];
                }
                st_row_chunk(sm + OFF_TW, r, j, tw, 1.f);
                st_row_chunk(sm + OFF_TU, r, j, tu, 1.f);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (s_abort) break;

        // ---- W^T = K^T (T diag(beta e^G))^T ; X = [T diag(beta); 0] V
        if (tid == 0) {
            if (mbar_wait(bar_v, n & 1, &failed)) {
                const uint32_t idw = idesc_bf16_f32(128, 64, true, false);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tW, sdesc_sw128(stage_a + k * 2048, 16384, 1024),
                             sdesc_sw128(sb + OFF_TW + k * 32, 16, 1024), idw, k > 0);
                const uint32_t idu = idesc_bf16_f32(128, 128, false, true);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tX, sdesc_sw128(sb + OFF_TU + k * 32, 16, 1024),
                             sdesc_sw128(sb + OFF_V + k * 2048, 8192, 1024), idu, k > 0);
            }
            mma_commit(bar_mma);
        }
        wait_all(bar_mma, mma_phase & 1);
        ++mma_phase;
        tc_fence_after();
        if (tid == 0 && n + 1 < NC) {
            fence_async_smem();
            load_v(n + 1);
        }
        // -W^T -> MN-major block 0 of WQ, row d = tid
        {
            float wv[64];
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_ld16(tW + lane_off + 16 * j, *reinterpret_cast<float(*)[16]>(wv + 16 * j));
            tmem_wait_ld();
            reg_fence(wv);
#pragma unroll
            for (int j = 0; j < 8; ++j) st_row_chunk(sm + OFF_WQ, tid, j, wv + 8 * j, -1.f);
        }
        // state -> bf16 h (MN-major [d][64 v] x 2), then state *= e^(G_C) in TMEM
        {
            const float gam = sGam[63];
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float hv[64];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    tmem_ld16(tH + lane_off + 64 * half + 16 * j, *reinterpret_cast<float(*)[16]>(hv + 16 * j));
                tmem_wait_ld();
                reg_fence(hv);
#pragma unroll
                for (int j = 0; j < 8; ++j) st_row_chunk(sm + OFF_HB + half * 16384, tid, j, hv + 8 * j, 1.f);
                if constexpr (GATE != kGateNone) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) hv[e] *= gam;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        tmem_st16(tH + lane_off + 64 * half + 16 * j, *reinterpret_cast<float(*)[16]>(hv + 16 * j));
                }
            }
            tmem_wait_st();
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (s_abort) break;

        // ---- X += [-W; Q_bar] h
        if (tid == 0) {
            const uint32_t id = idesc_bf16_f32(128, 128, true, true);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16(tX, sdesc_sw128(sb + OFF_WQ + k * 2048, 16384, 1024),
                         sdesc_sw128(sb + OFF_HB + k * 2048, 16384, 1024), id, true);
            mma_commit(bar_mma);
        }
        wait_all(bar_mma, mma_phase & 1);
        ++mma_phase;
        tc_fence_after();
        if (tid < 64) {   // D rows (lanes 0..63) -> D and D~ as MN-major [i][64 v] x 2
            const float ft = sFt[tid];
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float dv[64];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    tmem_ld16(tX + lane_off + 64 * half + 16 * j, *reinterpret_cast<float(*)[16]>(dv + 16 * j));
                tmem_wait_ld();
                reg_fence(dv);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    st_row_chunk(sm + OFF_DL + half * 8192, tid, j, dv + 8 * j, 1.f);
                    st_row_chunk(sm + OFF_DT + half * 8192, tid, j, dv + 8 * j, ft);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (s_abort) break;

        // ---- state += K^T D~ ; X += [0; P] D
        if (tid == 0) {
            const uint32_t id2 = idesc_bf16_f32(128, 128, true, true);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_bf16(tH, sdesc_sw128(stage_a + k * 2048, 16384, 1024),
                         sdesc_sw128(sb + OFF_DT + k * 2048, 8192, 1024), id2, true);
            const uint32_t id1 = idesc_bf16_f32(128, 128, false, true);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_bf16(tX, sdesc_sw128(sb + OFF_Z + k * 32, 16, 1024),
                         sdesc_sw128(sb + OFF_DL + k * 2048, 8192, 1024), id1, true);
            mma_commit(bar_mma);
        }
        wait_all(bar_mma, mma_phase & 1);
        ++mma_phase;
        tc_fence_after();
        if (tid >= 64) {   // O rows (lanes 64..127)
            const int r = tid - 64;
            __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + (((size_t)b * T + t0 + r) * H + h) * D;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float ov[64];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    tmem_ld16(tX + lane_off + 64 * half + 16 * j, *reinterpret_cast<float(*)[16]>(ov + 16 * j));
                tmem_wait_ld();
                reg_fence(ov);
                if (r < nval) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        uint4 w;
                        w.x = pack_bf16(ov[8 * j + 0], ov[8 * j + 1]);
                        w.y = pack_bf16(ov[8 * j + 2], ov[8 * j + 3]);
                        w.z = pack_bf16(ov[8 * j + 4], ov[8 * j + 5]);
                        w.w = pack_bf16(ov[8 * j + 6], ov[8 * j + 7]);
                        *reinterpret_cast<uint4*>(orow + 64 * half + 8 * j) = w;
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (s_abort) break;
    }

    if (!s_abort && p.s_out) {
        float* dst = p.s_out + ((size_t)bh * D + tid) * D;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            float hv[64];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                tmem_ld16(tH + lane_off + 64 * half + 16 * j, *reinterpret_cast<float(*)[16]>(hv + 16 * j));
            tmem_wait_ld();
            reg_fence(hv);
#pragma unroll
            for (int e = 0; e < 64; e += 4)
                *reinterpret_cast<float4*>(dst + 64 * half + e) = make_float4(hv[e], hv[e + 1], hv[e + 2], hv[e + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

bool make_maps(const ChunkParams& p, TcMaps* m) {
    const uint64_t dims[3] = {(uint64_t)p.H * D, (uint64_t)p.T, (uint64_t)p.B};
    const uint64_t strides[2] = {(uint64_t)p.H * D * 2, (uint64_t)p.T * p.H * D * 2};
    const uint32_t box[3] = {64, 64, 1};
    return make_tmap_bf16(&m->q, p.q, 3, dims, strides, box) &&
           make_tmap_bf16(&m->k, p.k, 3, dims, strides, box) &&
           make_tmap_bf16(&m->v, p.v, 3, dims, strides, box);
}

template <int GATE>
cudaError_t launch_gate(const ChunkParams& p, cudaStream_t s) {
    TcMaps maps;
    if (!make_maps(p, &maps)) return cudaErrorInvalidValue;
    auto kern = chunk_fwd_tc_kernel<GATE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)((size_t)p.B * p.H), NT, SMEM_BYTES, s>>>(maps, p);
    return cudaGetLastError();
}

}  // namespace

bool chunk_fwd_tc_supported(int Dk, int Dv, int gate) {
    return Dk == D && Dv == D && (gate == kGateNone || gate == kGateScalar);
}

cudaError_t launch_chunk_fwd_tc(const ChunkParams& p, int gate, cudaStream_t s) {
    if (gate == kGateScalar) return launch_gate<kGateScalar>(p, s);
    return launch_gate<kGateNone>(p, s);
}

}  // namespace gdn
