// osdn_precondition.cu -- phase 1 of the preconditioned delta rule: the O(d_k)
// scan over the key stream that yields the write keys kw_t = d_t (.) k_t.
//
// "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
// Attention", sec. 2.1 (right-preconditioning the gradient step by
// D_t = diag(d_t) is writing along kw_t = d_t (.) k_t), sec. 2.2 (d_t follows
// online gradient descent on the closed-form surrogate
// h_t(d) = ((1 - beta_t <d, k_t^2>)^2 - 1) / (2 |k_t|^2), which depends on the
// key and beta only), sec. 2.3 (a retention gate r_t scales d before the
// step).  Per (batch, head), token by token:
//     s = <d, k_t^2>,  n = |k_t|^2
//     kw_t = d (.) k_t
//     d   <- r_t d + eta beta_t (1 - beta_t s) k_t^2 / n      (d unchanged if n = 0)
// The scan is sequential in t and independent across (batch, head), so its
// time is the latency of one token times T.  Eight lanes share one head (each
// holds d_k / 8 components of d in registers): a token's two dot products take
// three butterfly steps.  The keys stream through shared memory: each lane
// copies its own slice of the next block of tokens (cp.async) while it works
// on the current block, so no global load is on the token-to-token path (a
// block spans a few microseconds of scan, longer than a load from memory);
// beta and r of a block are loaded one block ahead, eight tokens of four heads
// a load instruction, and broadcast by shuffles.
#include "common.cuh"

namespace gdn {
namespace {

constexpr int OSDN_WARPS = 2;              // warps per block; four heads a warp
constexpr int OSDN_THREADS = 32 * OSDN_WARPS;
constexpr int NBUF = 2;                    // blocks in flight per lane
// tokens per prefetch block: 2 KB of ring per lane for d_k = 128
template <typename Tin>
constexpr int tokens_per_block() { return sizeof(Tin) == 2 ? 32 : 16; }

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename Tin, int DK>
__global__ void __launch_bounds__(OSDN_THREADS)
osdn_precondition_kernel(const OsdnParams p) {
    constexpr int TB = tokens_per_block<Tin>();
    constexpr int NBR = TB / 8;                        // beta / r registers a lane per block
    constexpr int PL = DK / 8;                         // components of d per lane
    constexpr int LB = PL * (int)sizeof(Tin);          // bytes of a lane's slice of one key
    constexpr int NV = LB / 16;                        // 16-byte pieces of that slice
    static_assert(LB % 16 == 0, "slice of whole 16-byte pieces");
    extern __shared__ __align__(16) uint8_t stage_raw[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sub = lane & 7, hw = lane >> 3;
    const long long bh = ((long long)blockIdx.x * OSDN_WARPS + warp) * 4 + hw;
    const bool active = bh < (long long)p.B * p.H;
    const int b = active ? (int)(bh / p.H) : 0, h = active ? (int)(bh % p.H) : 0;
    const Tin* kp = static_cast<const Tin*>(p.k);
    const Tin* bp = static_cast<const Tin*>(p.beta);
    const Tin* rp = static_cast<const Tin*>(p.r);
    Tin* kwp = static_cast<Tin*>(p.kw);
    const int T = p.T;
    // this lane's ring: NBUF blocks of TB tokens, LB bytes each
    uint8_t* ring = stage_raw + (size_t)tid * NBUF * TB * LB;
    auto tok = [&](int t) { return ((long long)b * T + t) * p.H + h; };

    float d[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) d[i] = (active && p.d0) ? p.d0[bh * DK + sub * PL + i] : 1.f;

    // copy block `blk` (tokens TB blk ..) of this lane's key slices into its ring
    auto fetch_keys = [&](int blk) {
        if (active) {
            uint8_t* dst = ring + (blk % NBUF) * TB * LB;
#pragma unroll
            for (int i = 0; i < TB; ++i) {
                const int t = blk * TB + i;
                if (t < T) {
                    const uint8_t* src = reinterpret_cast<const uint8_t*>(kp + tok(t) * DK + sub * PL);
#pragma unroll
                    for (int j = 0; j < NV; ++j) cp_async16(dst + i * LB + 16 * j, src + 16 * j);
                }
            }
        }
        cp_async_commit();
    };
    // beta and r of block `blk`: register g of lane 4 i + hw' holds token
    // TB blk + 8 g + i of head hw' of this warp; every lane of a head reads its
    // token's value by shuffle
    const int hh = lane & 3;
    const long long bh2 = ((long long)blockIdx.x * OSDN_WARPS + warp) * 4 + hh;
    const bool act2 = bh2 < (long long)p.B * p.H;
    const int b2 = act2 ? (int)(bh2 / p.H) : 0, h2 = act2 ? (int)(bh2 % p.H) : 0;
    auto fetch_br = [&](int blk, float (&bt)[NBR], float (&rt)[NBR]) {
#pragma unroll
        for (int g = 0; g < NBR; ++g) {
            const int t = blk * TB + 8 * g + (lane >> 2);
            bt[g] = 0.f;
            rt[g] = 1.f;
            if (act2 && t < T) {
                const long long tk = ((long long)b2 * T + t) * p.H + h2;
                bt[g] = to_f32(bp[tk]);
                if (rp) rt[g] = to_f32(rp[tk]);
            }
        }
    };

    const int nblk = (T + TB - 1) / TB;
    float bcur[NBR], rcur[NBR], bnext[NBR], rnext[NBR];
#pragma unroll
    for (int g = 0; g < NBR; ++g) {
        bcur[g] = bnext[g] = 0.f;
        rcur[g] = rnext[g] = 1.f;
    }
    if (nblk > 0) {
        fetch_keys(0);
        fetch_br(0, bcur, rcur);
    }
#pragma unroll 1
    for (int blk = 0; blk < nblk; ++blk) {
        const bool more = blk + 1 < nblk;
        if (more) {
            fetch_keys(blk + 1);
            fetch_br(blk + 1, bnext, rnext);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncwarp();
        const uint8_t* src = ring + (blk % NBUF) * TB * LB;
#pragma unroll 1
        for (int i = 0; i < TB; ++i) {
            const int t = blk * TB + i;
            if (t >= T) break;   // uniform across the warp
            float kc[PL];
            {
                uint4 raw[NV];
#pragma unroll
                for (int j = 0; j < NV; ++j) raw[j] = *reinterpret_cast<const uint4*>(src + i * LB + 16 * j);
                const Tin* e = reinterpret_cast<const Tin*>(raw);
#pragma unroll
                for (int c = 0; c < PL; ++c) kc[c] = to_f32(e[c]);
            }
            float bsel = bcur[0], rsel = rcur[0];
#pragma unroll
            for (int g = 1; g < NBR; ++g) {
                if ((i >> 3) == g) {
                    bsel = bcur[g];
                    rsel = rcur[g];
                }
            }
            const float bt = __shfl_sync(0xffffffffu, bsel, 4 * (i & 7) + hw);
            const float rt = __shfl_sync(0xffffffffu, rsel, 4 * (i & 7) + hw);
            float s0 = 0.f, s1 = 0.f, n0 = 0.f, n1 = 0.f;
            float u[PL];
#pragma unroll
            for (int c = 0; c < PL; c += 2) {
                u[c] = kc[c] * kc[c];
                u[c + 1] = kc[c + 1] * kc[c + 1];
                s0 = fmaf(d[c], u[c], s0);
                s1 = fmaf(d[c + 1], u[c + 1], s1);
                n0 += u[c];
                n1 += u[c + 1];
            }
            float s = s0 + s1, n = n0 + n1;
#pragma unroll
            for (int off = 1; off < 8; off <<= 1) {
                s += __shfl_xor_sync(0xffffffffu, s, off);
                n += __shfl_xor_sync(0xffffffffu, n, off);
            }
            if (active) {
                uint4 raw[NV];
                Tin* e = reinterpret_cast<Tin*>(raw);
#pragma unroll
                for (int c = 0; c < PL; ++c) e[c] = from_f32<Tin>(d[c] * kc[c]);
                uint4* dst = reinterpret_cast<uint4*>(kwp + tok(t) * DK + sub * PL);
#pragma unroll
                for (int j = 0; j < NV; ++j) dst[j] = raw[j];
            }
            const float ef = n > 0.f ? p.eta * bt * (1.f - bt * s) / n : 0.f;
#pragma unroll
            for (int c = 0; c < PL; ++c) d[c] = fmaf(rt, d[c], ef * u[c]);
        }
        __syncwarp();   // every lane is done with this block's slot before it is refilled
#pragma unroll
        for (int g = 0; g < NBR; ++g) {
            bcur[g] = bnext[g];
            rcur[g] = rnext[g];
        }
    }
    if (active && p.d_out) {
#pragma unroll
        for (int c = 0; c < PL; ++c) p.d_out[bh * DK + sub * PL + c] = d[c];
    }
}

template <typename Tin, int DK>
cudaError_t launch_dk(const OsdnParams& p, cudaStream_t s) {
    const long long nbh = (long long)p.B * p.H;
    const int heads_per_block = 4 * OSDN_WARPS;
    const unsigned grid = (unsigned)((nbh + heads_per_block - 1) / heads_per_block);
    const size_t smem = (size_t)OSDN_THREADS * NBUF * tokens_per_block<Tin>() * (DK / 8) * sizeof(Tin);
    auto kern = osdn_precondition_kernel<Tin, DK>;
    if (smem > 48 * 1024) {
        const cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_on(kern, dim3(grid), dim3(OSDN_THREADS), smem, s, p);
}

}  // namespace

cudaError_t launch_osdn_precondition(const OsdnParams& p, int Dk, bool bf16, cudaStream_t s) {
    if (bf16) return Dk == 64 ? launch_dk<__nv_bfloat16, 64>(p, s) : launch_dk<__nv_bfloat16, 128>(p, s);
    return Dk == 64 ? launch_dk<float, 64>(p, s) : launch_dk<float, 128>(p, s);
}

}  // namespace gdn
