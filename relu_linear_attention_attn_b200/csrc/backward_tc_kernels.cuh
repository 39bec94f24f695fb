// The key side of the backward of Eq. (1) ("Sana: Efficient High-Resolution Image
// Synthesis with Linear Diffusion Transformers", section 2.1) with the per-head
// QK-RMSNorm feature map of "SANA 1.5 ...", section "Model architecture", on the
// tensor cores (bf16 inputs and outputs, fp32 accumulation).  With the gradient
// state [dS | dz] of every (b, h) (dS[d][e] = sum_t phi(Q)_t[d] dnum_t[e],
// dz[d] = sum_t phi(Q)_t[d] dden_t), per key token t and head h:
//     dV_t[e]      = sum_d phi(K)_t[d] dS[d][e]
//     dphi(K)_t[d] = sum_e dS[d][e] V_t[e] + dz[d]
// then the feature map's backward gives dK and the per-channel gain gradient.
//
// bwd_key_tc: work item = one 128-token tile of one row (b, head pair), persistent
// CTAs over a balanced flat list as in the forward's pass 2.  Per row segment a
// builder warp writes two B operands per head from [dS | dz] (fp32, read from
// global memory), K-major, 64 rows each: rows 0..31 the bf16 "hi" parts, rows
// 32..63 the "lo" parts (x - bf16(x)), so one UMMA covers both:
//     Bop1[n = e][k = d] = dS[d][e]        (for dV)
//     Bop2[n = d][k = e] = dS[d][e]        (for dphi(K))
// The workers rewrite the K tile in place as ReLU(g k) (r = 1/rms kept in a
// register; the gains read from global memory, 16-byte aligned, so that shared
// memory holds six stages); per head two UMMAs each (M = 128, N = 64, K = 16)
//     D1 = ReLU(g k) Bop1,   D2 = V Bop2        (V straight from its tile, K-major)
// and the epilogue forms dV = r (D1[e] + D1[32 + e]) over the V tile, dphi(K) =
// D2[d] + D2[32 + d] + dz[d], the feature map's backward with the raw k row (read
// again from global memory) over the K tile, and a store warp TMA-stores both.
// Gain gradients: each warp's 32 rows are summed per channel (butterfly) and
// written per (tile, quadrant, head); `gain_combine_tiles` and
// `gain_combine_slices` sum them in a fixed order, so the result is reproducible.
//
// TMEM: warp w reads lanes 32 * (w % 4) .. + 31; D row i is lane i.
#pragma once

#include "sana_common.cuh"
#include "sm100_primitives.cuh"
#include "tc_kernels.cuh"

namespace sana {

namespace bk {
constexpr int kTileTok = 128;                      // UMMA M
constexpr int kTileBytes = kTileTok * 128;         // 128 tokens x 64 channels (a head pair)
constexpr int kStageBytes = 2 * kTileBytes;        // [K | V]
constexpr int kStages = 6;
constexpr int kN = 64;                             // B rows per head: 32 hi, 32 lo
constexpr int kBopBytes = kN * 128;                // both heads side by side in each row
constexpr int kBopSet = 2 * kBopBytes;             // Bop1, Bop2 of a row segment
constexpr int kBopRing = 2;
constexpr int kBufCols = 4 * kN;                   // [D1 head 0 | D1 head 1 | D2 head 0 | D2 head 1]
constexpr int kTmemCols = 2 * kBufCols;            // one buffer per tile group
constexpr int kWorkerWarps = 16;                   // two tile groups of 8
constexpr int kGroupThreads = 32 * kWorkerWarps / 2;
constexpr int kThreads = 32 * (4 + kWorkerWarps);  // TMA, UMMA, builder, store, workers
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kBopRing * kBopSet + 1024;
// (A slot may serve the two worker groups in turn: a group's use of slot s for tile
// li + kStages starts after the tile in it before, li, has been stored, so the
// per-slot barriers never see two tiles' arrivals at once.)
static_assert(kTmemCols <= 512, "TMEM");
static_assert(kSmemBytes <= 232448, "shared memory");
}  // namespace bk

// The feature map's backward for one row of one head, in place: dp holds dphi on
// entry (fp32), raw the row's 32 bf16 inputs (packed pairs), g its gains (norm on), r
// its 1/rms.  du = dphi where g x r > 0 (x > 0 with the norm off);
//   dx = g r du - r^3 (sum_u du g x / D) x        (norm on; dx = du with the norm off)
// dx goes out as bf16 to the swizzled row `dst` (4 chunks from chunk0), and dp
// returns the gain gradient's share du x r (zeros with the norm off or a dead row).
__device__ __forceinline__ void phi_bwd_row(float* dp, const uint4 raw[4], const float* g, float r,
                                            bool norm, bool live, uint8_t* tile, int row, int chunk0) {
    auto xr = [&](int u) -> float {
        const uint4 w4 = raw[u >> 3];
        const int k = (u >> 1) & 3;
        const uint32_t w = k == 0 ? w4.x : k == 1 ? w4.y : k == 2 ? w4.z : w4.w;
        return (u & 1) ? bf16hi(w) : bf16lo(w);
    };
    float cf = 0.f;
    if (norm) {
        float tsum = 0.f;
#pragma unroll
        for (int u = 0; u < kD; ++u) {
            const float x = xr(u), gu = g[u];
            dp[u] = gu * x > 0.f ? dp[u] : 0.f;                   // du
            tsum = fmaf(dp[u] * gu, x, tsum);
        }
        cf = r * r * r * tsum * (1.f / kD);
    } else {
#pragma unroll
        for (int u = 0; u < kD; ++u) dp[u] = xr(u) > 0.f ? dp[u] : 0.f;
    }
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
        float o[8];
#pragma unroll
        for (int u8 = 0; u8 < 8; ++u8) {
            const int u = 8 * cc + u8;
            const float x = xr(u), du = dp[u];
            o[u8] = norm ? g[u] * r * du - cf * x : du;
            dp[u] = norm ? du * x * r : 0.f;                       // gain share
        }
        uint4 w;
        w.x = pack_bf16x2(o[0], o[1]);
        w.y = pack_bf16x2(o[2], o[3]);
        w.z = pack_bf16x2(o[4], o[5]);
        w.w = pack_bf16x2(o[6], o[7]);
        if (!live) w = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(tile + sw128_offset(row, chunk0 + cc)) = w;
    }
    if (!live) {
#pragma unroll
        for (int u = 0; u < kD; ++u) dp[u] = 0.f;
    }
}

struct BkArgs {
    const float* dsz;    // [dS | dz]: [B][H][D][D+1]
    const float* gk;     // gains [C] or nullptr (norm off)
    const bf16* k;       // raw keys (B, N, C), for the feature map's backward
    float* gpart;        // gain partials [T][4 quadrants][2 heads][D] (norm on)
    int64_t T;           // work items: B * Pp rows x R tiles
    int N, H, Pp, R, P;
    float eps;
    int norm;
};

__global__ void __launch_bounds__(bk::kThreads, 1)   // 640 threads: at most 96 registers
bwd_key_tc(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
           const __grid_constant__ CUtensorMap tmap_dk, const __grid_constant__ CUtensorMap tmap_dv,
           const BkArgs a)
{
    using namespace bk;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* stages = smem;
    uint8_t* bop = stages + kStages * kStageBytes;
    uint64_t* full = (uint64_t*)(bop + kBopRing * kBopSet);
    uint64_t* aready = full + kStages;
    uint64_t* mmadone = aready + kStages;
    uint64_t* tready = mmadone + kStages;
    uint64_t* empty = tready + kStages;
    uint64_t* tfree = empty + kStages;                  // 2: one per tile group
    uint64_t* bfull = tfree + 2;
    uint64_t* bempty = bfull + kBopRing;
    uint64_t* drain = bempty + kBopRing;
    uint32_t* tmem_slot = (uint32_t*)(drain + 1);

    const int64_t c = blockIdx.x;
    const int64_t i0 = range_begin(c, a.T, a.P), i1 = range_begin(c + 1, a.T, a.P);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&aready[i], kGroupThreads);
            mbar_init(&mmadone[i], 1);
            mbar_init(&tready[i], kGroupThreads);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) mbar_init(&tfree[i], kGroupThreads);
        for (int i = 0; i < kBopRing; ++i) {
            mbar_init(&bfull[i], 32);
            mbar_init(&bempty[i], 1);
        }
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
        prefetch_tmap(&tmap_dk);
        prefetch_tmap(&tmap_dv);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // [dS | dz] and the keys' gradients come from earlier launches on this stream
    pdl_wait_primary();
    bool ok = i1 > i0;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (K and V tiles)
        if (lane == 0 && ok) {
            int64_t last = -1;
            for (int64_t li = 0; i0 + li < i1; ++li) {
                const int st = (int)(li % kStages);
                if (li >= kStages) ok = mbar_wait(&empty[st], (uint32_t)((li / kStages) - 1) & 1, 601);
                if (!ok) break;
                const int64_t i = i0 + li, r = i / a.R;
                const int t = (int)(i % a.R), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
                uint8_t* sb = stages + st * kStageBytes;
                mbar_arrive_expect_tx(&full[st], kStageBytes);
                tma_load_3d(sb, &tmap_k, &full[st], p * 64, t * kTileTok, b);
                tma_load_3d(sb + kTileBytes, &tmap_v, &full[st], p * 64, t * kTileTok, b);
                last = li;
            }
            if (!ok) {   // let every issued copy land before the CTA can exit
                for (int64_t lj = last - (kStages - 1) > 0 ? last - (kStages - 1) : 0; lj <= last; ++lj)
                    mbar_wait(&full[lj % kStages], (uint32_t)(lj / kStages) & 1, 602);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer (lane 0 alone)
        if (ok && lane == 0) {
            const uint32_t idesc = make_idesc_bf16(128, kN, false, false);
            const uint64_t s0 = make_smem_desc(smem_u32(stages), 16, 1024, kSwizzle128B);
            const uint64_t b0 = make_smem_desc(smem_u32(bop), 16, 1024, kSwizzle128B);
            const int64_t n = i1 - i0;
            int seg = 0;
            int64_t t = i0 % a.R;
            for (int64_t li = 0; li < n && ok; ++li) {
                const bool first = (li == 0) || (t == 0);
                const bool lastt = (li + 1 == n) || (t == a.R - 1);
                const int st = (int)(li % kStages), tb = (int)(li & 1), rb = seg & 1;
                if (first) ok = mbar_wait(&bfull[rb], (uint32_t)(seg >> 1) & 1, 603);
                if (ok) ok = mbar_wait(&aready[st], (uint32_t)(li / kStages) & 1, 604);
                if (ok && li >= 2) ok = mbar_wait(&tfree[tb], (uint32_t)((li >> 1) - 1) & 1, 605);
                if (!ok) break;
                tc_fence_after_sync();
                const uint64_t kd = s0 + (uint64_t)((st * kStageBytes) >> 4);
                const uint64_t vd = kd + (uint64_t)(kTileBytes >> 4);
                const uint64_t b1 = b0 + (uint64_t)((rb * kBopSet) >> 4);
                const uint64_t b2 = b1 + (uint64_t)(kBopBytes >> 4);
                const uint32_t d = tmem + tb * kBufCols;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    umma_bf16(d + j * kN, kd + 4 * j, b1 + 4 * j, idesc, false);
                    umma_bf16(d + j * kN, kd + 4 * j + 2, b1 + 4 * j + 2, idesc, true);
                    umma_bf16(d + (2 + j) * kN, vd + 4 * j, b2 + 4 * j, idesc, false);
                    umma_bf16(d + (2 + j) * kN, vd + 4 * j + 2, b2 + 4 * j + 2, idesc, true);
                }
                umma_commit(&mmadone[st]);
                if (lastt) {
                    umma_commit(&bempty[rb]);
                    ++seg;
                }
                if (++t == a.R) t = 0;
            }
            umma_commit(drain);
            mbar_wait(drain, 0, 606);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------------------------ B operands of each row segment
        // lane = d: the row dS[d][0..31] and dz[d] of each head of the pair
        int seg = 0;
        for (int64_t li = 0; i0 + li < i1 && ok; ++li) {
            const int64_t i = i0 + li;
            if (!(li == 0 || i % a.R == 0)) continue;              // not a segment start
            const int rb = seg & 1;
            if (seg >= 2) ok = mbar_wait(&bempty[rb], (uint32_t)((seg >> 1) - 1) & 1, 607);
            if (!ok) break;
            const int64_t r = i / a.R;
            const int b = (int)(r / a.Pp), p = (int)(r % a.Pp);
            const int h0 = 2 * p, nh = min(2, a.H - h0);
            uint8_t* b1 = bop + rb * kBopSet;
            uint8_t* b2 = b1 + kBopBytes;
            const int d0 = lane & ~1;
#pragma unroll 1
            for (int j = 0; j < 2; ++j) {
                float x[kD];
                const float* src = a.dsz + ((size_t)b * a.H + h0 + j) * kStateFloats + lane * kDP;
#pragma unroll
                for (int e = 0; e < kD; ++e) x[e] = j < nh ? __ldg(src + e) : 0.f;
                // Bop2: row n = d (this lane), K = e: lanes write their own rows, pairs of e
#pragma unroll
                for (int e = 0; e < kD; e += 2) {
                    const float h_0 = __bfloat162float(__float2bfloat16_rn(x[e]));
                    const float h_1 = __bfloat162float(__float2bfloat16_rn(x[e + 1]));
                    const int chunk = j * 4 + e / 8, off = (e % 8) * 2;
                    *reinterpret_cast<uint32_t*>(b2 + sw128_offset(lane, chunk) + off) = pack_bf16x2(h_0, h_1);
                    *reinterpret_cast<uint32_t*>(b2 + sw128_offset(kD + lane, chunk) + off) =
                        pack_bf16x2(x[e] - h_0, x[e + 1] - h_1);
                }
                // Bop1: row n = e, K = d: lane pairs (d, d + 1) write one bf16x2 each, even
                // lanes the hi part, odd lanes the lo part
                const int chunk = j * 4 + d0 / 8, off = (d0 % 8) * 2;
#pragma unroll
                for (int e = 0; e < kD; ++e) {
                    const float xv = x[e];
                    const float xp = __shfl_xor_sync(0xffffffffu, xv, 1);
                    const float xe = (lane & 1) ? xp : xv, xo = (lane & 1) ? xv : xp;
                    const float he = __bfloat162float(__float2bfloat16_rn(xe));
                    const float ho = __bfloat162float(__float2bfloat16_rn(xo));
                    const int row = (lane & 1) ? kD + e : e;
                    const uint32_t w = (lane & 1) ? pack_bf16x2(xe - he, xo - ho) : pack_bf16x2(he, ho);
                    *reinterpret_cast<uint32_t*>(b1 + sw128_offset(row, chunk) + off) = w;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            mbar_arrive(&bfull[rb]);
            ++seg;
        }
    } else if (warp == 3) {
        // ------------------------------------------------ dK, dV stores (over the K, V tiles)
        if (lane == 0 && ok) {
            int64_t li = 0;
            for (; i0 + li < i1 && ok; ++li) {
                const int st = (int)(li % kStages);
                ok = mbar_wait(&tready[st], (uint32_t)(li / kStages) & 1, 608);
                if (!ok) break;
                const int64_t i = i0 + li, r = i / a.R;
                const int t = (int)(i % a.R), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
                uint8_t* sb = stages + st * kStageBytes;
                tma_store_3d(&tmap_dk, sb, p * 64, t * kTileTok, b);
                tma_store_3d(&tmap_dv, sb + kTileBytes, p * 64, t * kTileTok, b);
                bulk_commit_group();
                bulk_wait_group_read<0>();
                mbar_arrive(&empty[st]);
            }
            bulk_wait_group<0>();
        }
    } else {
        // ------------------------------------------------ ReLU(g k), then the epilogue
        // Two tile groups of 8 warps take alternate tiles; in a group, warp w takes TMEM
        // quadrant w % 4 (token rows 32 (w % 4) ..) and head (w / 4) % 2 of the pair.
        const int wi = warp - 4;                          // 0..15
        const int grp = wi >> 3;                          // tiles with li % 2 == grp
        const int j = (wi >> 2) & 1;                      // head of the pair
        const int q = warp & 3;                           // TMEM lane quadrant
        const int row = 32 * q + lane;                    // token row of the tile
        auto transform = [&](int64_t li, float& rk) -> bool {
            const int st = (int)(li % kStages);
            if (!mbar_wait(&full[st], (uint32_t)(li / kStages) & 1, 609)) return false;
            const int64_t i = i0 + li, r = i / a.R;
            const int t = (int)(i % a.R), p = (int)(r % a.Pp);
            const int h = p * 2 + j;
            const bool live = (t * kTileTok + row < a.N) && h < a.H;
            rk = phi_inplace_sw128<false>(stages + st * kStageBytes, row, j * 4,
                                          a.norm ? a.gk + (live ? h : 0) * kD : nullptr, a.eps,
                                          a.norm != 0, !live);
            fence_proxy_async_smem();
            mbar_arrive(&aready[st]);
            return true;
        };
        auto epilogue = [&](int64_t li, float rk) -> bool {
            const int st = (int)(li % kStages), tb = (int)(li & 1);
            if (!mbar_wait(&mmadone[st], (uint32_t)(li / kStages) & 1, 610)) return false;
            tc_fence_after_sync();
            const int64_t i = i0 + li, r = i / a.R;
            const int t = (int)(i % a.R), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
            const int h = p * 2 + j;
            const int64_t tok = (int64_t)t * kTileTok + row;
            const bool live = tok < a.N && h < a.H;
            uint8_t* ktile = stages + st * kStageBytes;
            uint8_t* vtile = ktile + kTileBytes;
            const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + tb * kBufCols;
            // the raw k row for the feature map's backward, requested first so that its
            // latency overlaps the TMEM work below
            uint4 kraw[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                             make_uint4(0, 0, 0, 0)};
            if (live) {
                const uint4* kr = reinterpret_cast<const uint4*>(
                    a.k + ((size_t)b * a.N + tok) * (size_t)(a.H * kD) + (size_t)h * kD);
#pragma unroll
                for (int u = 0; u < 4; ++u) kraw[u] = __ldg(kr + u);
            }
            // dV = r (D1 hi + lo), over this head's columns of the V tile (V was read by
            // the UMMA that completed mmadone)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float hi[16], lo[16];
                tmem_ld16(ta + j * kN + 16 * hf, hi);
                tmem_ld16(ta + j * kN + kD + 16 * hf, lo);
                tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    float o[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) o[u] = (hi[8 * cc + u] + lo[8 * cc + u]) * rk;
                    uint4 w;
                    w.x = pack_bf16x2(o[0], o[1]);
                    w.y = pack_bf16x2(o[2], o[3]);
                    w.z = pack_bf16x2(o[4], o[5]);
                    w.w = pack_bf16x2(o[6], o[7]);
                    *reinterpret_cast<uint4*>(vtile + sw128_offset(row, j * 4 + 2 * hf + cc)) = w;
                }
            }
            // dphi(K) = D2 hi + lo + dz (dz from global memory: the builder's ring slot may
            // already hold a later segment's operands)
            float dp[kD];
            const float* dz = a.dsz + ((size_t)b * a.H + (h < a.H ? h : 0)) * kStateFloats + kD;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float hi[16], lo[16];
                tmem_ld16(ta + (2 + j) * kN + 16 * hf, hi);
                tmem_ld16(ta + (2 + j) * kN + kD + 16 * hf, lo);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; ++u) dp[16 * hf + u] = (hi[u] + lo[u]) + __ldg(dz + (16 * hf + u) * kDP);
            }
            tc_fence_before_sync();
            mbar_arrive(&tfree[tb]);
            // the feature map's backward with the raw k row -> dK over the K tile
            phi_bwd_row(dp, kraw, a.norm ? a.gk + (h < a.H ? h : 0) * kD : nullptr, rk, a.norm != 0,
                        live, ktile, row, j * 4);
            fence_proxy_async_smem();
            mbar_arrive(&tready[st]);
            if (a.norm) {                                 // the warp's 32 rows, per channel
                warp_reduce_scatter32(dp, lane);
                a.gpart[((size_t)i * 4 + q) * (2 * kD) + j * kD + lane] = dp[0];
            }
            return true;
        };

        int64_t prev = -1;
        float r_prev = 1.f, r_cur = 1.f;
        for (int64_t li = grp; i0 + li < i1 && ok; li += 2) {
            ok = transform(li, r_cur);
            if (ok && prev >= 0) ok = epilogue(prev, r_prev);
            prev = li;
            r_prev = r_cur;
        }
        if (ok && prev >= 0) ok = epilogue(prev, r_prev);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ============================================================================ query side
// bwd_query_tc: the query side of the backward, per (b, head pair, 128-token tile).
// With the forward state S = [S_v | z] of every (b, h):
//     num = phi(Q) S_v, den = phi(Q) z, O = num / (den + eps)
//     dnum = dO / (den + eps),  dden = -(dO . O) / (den + eps)
//     dphi(Q)[d] = sum_e S_v[d][e] dnum[e] + z[d] dden
// then the feature map's backward gives dQ and the per-channel gain gradient.
// Per row segment a builder warp writes, per head, pass 2's B operand of S (80
// rows: value columns hi, normaliser hi / lo, value columns lo; U1) and the
// transposed state's (64 rows: S_v[d][.] hi, then lo; U2).  Per tile:
//   transform: ReLU(g q) in place in the Q tile (r = 1/rms kept in a register)
//   U1:        D = ReLU(g q) BopS                    (M = 128, N = 80, K = 16) x 2 per head
//   epilogue A: num, den (times r), O, dnum (bf16, over the dO tile: the A operand
//              of U2 and the dnum output), dden (fp32 output, and kept)
//   U2:        D = dnum BopT                          (N = 64) x 2 per head, over U1's columns
//   epilogue B: dphi(Q) = hi + lo + dden z, the feature map's backward with the raw q
//              row -> dQ over the Q tile; gain partials as in bwd_key_tc
// The issuer runs U1 of the next tile (the other worker group's) before U2 of the
// current one; each worker group runs A(li), the transform of its next tile, then
// B(li), so the UMMA latencies hide behind the other work.
namespace bq {
constexpr int kTileTok = 128;
constexpr int kTileBytes = kTileTok * 128;
constexpr int kStageBytes = 2 * kTileBytes;        // [Q | dO]
constexpr int kStages = 5;
constexpr int kNS = p2::kN;                        // 80: pass 2's operand of S
constexpr int kNT = 64;                            // S_v^T: 32 hi, 32 lo
constexpr int kBopSBytes = kNS * 128;
constexpr int kBopTBytes = kNT * 128;
constexpr int kBopSet = kBopSBytes + kBopTBytes;
constexpr int kBopRing = 2;
constexpr int kBufCols = 256;                      // per tile group: U1's 2 x 80, then U2's over it
constexpr int kTmemCols = 2 * kBufCols;
constexpr int kWorkerWarps = 16;
constexpr int kGroupThreads = 32 * kWorkerWarps / 2;
constexpr int kThreads = 32 * (4 + kWorkerWarps);
constexpr int kGainCache = 4096;
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kBopRing * kBopSet + kGainCache * 4 + 1024;
static_assert(kBopSBytes % 1024 == 0 && kBopSet % 1024 == 0, "operand alignment");
static_assert(kSmemBytes <= 232448, "shared memory");
}  // namespace bq

struct BqArgs {
    const float* s;      // forward states [B][H][D][D+1]
    const float* gq;     // gains [C] or nullptr (norm off)
    const bf16* q;       // raw queries, for the feature map's backward
    float* dden;         // [B][H][N] output
    float* gpart;        // gain partials [T][4 quadrants][2 heads][D] (norm on)
    int64_t T;
    int N, H, Pp, R, P;
    float eps;
    int norm;
};

__global__ void __launch_bounds__(bq::kThreads, 1)   // 640 threads: at most 96 registers
bwd_query_tc(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_do,
             const __grid_constant__ CUtensorMap tmap_dq, const __grid_constant__ CUtensorMap tmap_dnum,
             const BqArgs a)
{
    using namespace bq;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* stages = smem;
    uint8_t* bop = stages + kStages * kStageBytes;
    float* sgain = (float*)(bop + kBopRing * kBopSet);
    uint64_t* full = (uint64_t*)(sgain + kGainCache);
    uint64_t* aready = full + kStages;
    uint64_t* mma1 = aready + kStages;
    uint64_t* pready = mma1 + kStages;
    uint64_t* mma2 = pready + kStages;
    uint64_t* tready = mma2 + kStages;
    uint64_t* empty = tready + kStages;
    uint64_t* tfree = empty + kStages;                  // 2: one per tile group
    uint64_t* bfull = tfree + 2;
    uint64_t* bempty = bfull + kBopRing;
    uint64_t* drain = bempty + kBopRing;
    uint32_t* tmem_slot = (uint32_t*)(drain + 1);

    const int64_t c = blockIdx.x;
    const int64_t i0 = range_begin(c, a.T, a.P), i1 = range_begin(c + 1, a.T, a.P);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = a.H * kD;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&aready[i], kGroupThreads);
            mbar_init(&mma1[i], 1);
            mbar_init(&pready[i], kGroupThreads);
            mbar_init(&mma2[i], 1);
            mbar_init(&tready[i], kGroupThreads);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) mbar_init(&tfree[i], kGroupThreads);
        for (int i = 0; i < kBopRing; ++i) {
            mbar_init(&bfull[i], 32);
            mbar_init(&bempty[i], 1);
        }
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_do);
        prefetch_tmap(&tmap_dq);
        prefetch_tmap(&tmap_dnum);
    }
    // rows of pass 2's operand that never carry data stay zero
    for (int i = threadIdx.x; i < kBopRing * (p2::kLoRow - p2::kDenLo - 1) * 8; i += blockDim.x) {
        const int rb = i / ((p2::kLoRow - p2::kDenLo - 1) * 8), rem = i % ((p2::kLoRow - p2::kDenLo - 1) * 8);
        *reinterpret_cast<uint4*>(bop + rb * kBopSet + (p2::kDenLo + 1 + rem / 8) * 128 + (rem % 8) * 16) =
            make_uint4(0, 0, 0, 0);
    }
    if (a.norm) load_gains<bq::kGainCache, bq::kThreads>(sgain, a.gq, C, threadIdx.x);
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    pdl_wait_primary();                                 // the states come from earlier launches
    bool ok = i1 > i0;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (Q and dO tiles)
        if (lane == 0 && ok) {
            int64_t last = -1;
            for (int64_t li = 0; i0 + li < i1; ++li) {
                const int st = (int)(li % kStages);
                if (li >= kStages) ok = mbar_wait(&empty[st], (uint32_t)((li / kStages) - 1) & 1, 701);
                if (!ok) break;
                const int64_t i = i0 + li, r = i / a.R;
                const int t = (int)(i % a.R), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
                uint8_t* sb = stages + st * kStageBytes;
                mbar_arrive_expect_tx(&full[st], kStageBytes);
                tma_load_3d(sb, &tmap_q, &full[st], p * 64, t * kTileTok, b);
                tma_load_3d(sb + kTileBytes, &tmap_do, &full[st], p * 64, t * kTileTok, b);
                last = li;
            }
            if (!ok) {
                for (int64_t lj = last - (kStages - 1) > 0 ? last - (kStages - 1) : 0; lj <= last; ++lj)
                    mbar_wait(&full[lj % kStages], (uint32_t)(lj / kStages) & 1, 702);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer (lane 0 alone):
        // U1(0), then per tile li: U1(li + 1), U2(li)
        if (ok && lane == 0) {
            const uint32_t idesc_s = make_idesc_bf16(128, kNS, false, false);
            const uint32_t idesc_t = make_idesc_bf16(128, kNT, false, false);
            const uint64_t s0 = make_smem_desc(smem_u32(stages), 16, 1024, kSwizzle128B);
            const uint64_t b0 = make_smem_desc(smem_u32(bop), 16, 1024, kSwizzle128B);
            const int64_t n = i1 - i0;
            int seg1 = 0, seg2 = 0;                        // row segments seen by U1 / finished by U2
            int64_t t1 = i0 % a.R, t2 = i0 % a.R;
            auto u1 = [&](int64_t li) -> bool {
                const bool first = (li == 0) || (t1 == 0);
                const int st = (int)(li % kStages), tb = (int)(li & 1);
                if (first && !mbar_wait(&bfull[seg1 & 1], (uint32_t)(seg1 >> 1) & 1, 703)) return false;
                const int rb = seg1 & 1;
                if (!mbar_wait(&aready[st], (uint32_t)(li / kStages) & 1, 704)) return false;
                if (li >= 2 && !mbar_wait(&tfree[tb], (uint32_t)((li >> 1) - 1) & 1, 705)) return false;
                tc_fence_after_sync();
                const uint64_t qd = s0 + (uint64_t)((st * kStageBytes) >> 4);
                const uint64_t bs = b0 + (uint64_t)((rb * kBopSet) >> 4);
                const uint32_t d = tmem + tb * kBufCols;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    umma_bf16(d + j * kNS, qd + 4 * j, bs + 4 * j, idesc_s, false);
                    umma_bf16(d + j * kNS, qd + 4 * j + 2, bs + 4 * j + 2, idesc_s, true);
                }
                umma_commit(&mma1[st]);
                if ((li + 1 == n) || (t1 == a.R - 1)) ++seg1;
                if (++t1 == a.R) t1 = 0;
                return true;
            };
            auto u2 = [&](int64_t li) -> bool {
                const int st = (int)(li % kStages), tb = (int)(li & 1), rb = seg2 & 1;
                if (!mbar_wait(&pready[st], (uint32_t)(li / kStages) & 1, 706)) return false;
                tc_fence_after_sync();
                const uint64_t gd = s0 + (uint64_t)((st * kStageBytes + kTileBytes) >> 4);
                const uint64_t bt = b0 + (uint64_t)((rb * kBopSet + kBopSBytes) >> 4);
                const uint32_t d = tmem + tb * kBufCols;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    umma_bf16(d + j * kNS, gd + 4 * j, bt + 4 * j, idesc_t, false);
                    umma_bf16(d + j * kNS, gd + 4 * j + 2, bt + 4 * j + 2, idesc_t, true);
                }
                umma_commit(&mma2[st]);
                if ((li + 1 == n) || (t2 == a.R - 1)) {
                    umma_commit(&bempty[rb]);
                    ++seg2;
                }
                if (++t2 == a.R) t2 = 0;
                return true;
            };
            ok = u1(0);
            for (int64_t li = 0; li < n && ok; ++li) {
                if (li + 1 < n) ok = u1(li + 1);
                if (ok) ok = u2(li);
            }
            umma_commit(drain);
            mbar_wait(drain, 0, 707);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------------------------ B operands of each row segment;
        // lane = d: the row S[d][0..32] of each head of the pair
        int seg = 0;
        for (int64_t li = 0; i0 + li < i1 && ok; ++li) {
            const int64_t i = i0 + li;
            if (!(li == 0 || i % a.R == 0)) continue;
            const int rb = seg & 1;
            if (seg >= 2) ok = mbar_wait(&bempty[rb], (uint32_t)((seg >> 1) - 1) & 1, 708);
            if (!ok) break;
            const int64_t r = i / a.R;
            const int b = (int)(r / a.Pp), p = (int)(r % a.Pp);
            const int h0 = 2 * p, nh = min(2, a.H - h0);
            uint8_t* bs = bop + rb * kBopSet;
            uint8_t* bt = bs + kBopSBytes;
            const int d0 = lane & ~1;
#pragma unroll 1
            for (int j = 0; j < 2; ++j) {
                float x[kDP];
                const float* src = a.s + ((size_t)b * a.H + h0 + j) * kStateFloats + lane * kDP;
#pragma unroll
                for (int e = 0; e < kDP; ++e) x[e] = j < nh ? __ldg(src + e) : 0.f;
                // pass 2's operand: row e (value column) / 32, 33 (normaliser) hi, lo
                const int chunk = j * 4 + d0 / 8, off = (d0 % 8) * 2;
#pragma unroll
                for (int e = 0; e < kDP; ++e) {
                    const float xv = x[e];
                    const float xp = __shfl_xor_sync(0xffffffffu, xv, 1);
                    const float xe = (lane & 1) ? xp : xv, xo = (lane & 1) ? xv : xp;
                    const float he = __bfloat162float(__float2bfloat16_rn(xe));
                    const float ho = __bfloat162float(__float2bfloat16_rn(xo));
                    const int row = (lane & 1) ? (e < kD ? p2::kLoRow + e : p2::kDenLo) : e;
                    const uint32_t w = (lane & 1) ? pack_bf16x2(xe - he, xo - ho) : pack_bf16x2(he, ho);
                    *reinterpret_cast<uint32_t*>(bs + sw128_offset(row, chunk) + off) = w;
                }
                // the transposed state: row n = d (this lane), K = e
#pragma unroll
                for (int e = 0; e < kD; e += 2) {
                    const float h_0 = __bfloat162float(__float2bfloat16_rn(x[e]));
                    const float h_1 = __bfloat162float(__float2bfloat16_rn(x[e + 1]));
                    const int ck = j * 4 + e / 8, of = (e % 8) * 2;
                    *reinterpret_cast<uint32_t*>(bt + sw128_offset(lane, ck) + of) = pack_bf16x2(h_0, h_1);
                    *reinterpret_cast<uint32_t*>(bt + sw128_offset(kD + lane, ck) + of) =
                        pack_bf16x2(x[e] - h_0, x[e + 1] - h_1);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            mbar_arrive(&bfull[rb]);
            ++seg;
        }
    } else if (warp == 3) {
        // ------------------------------------------------ dQ, dnum stores (over Q, dO tiles)
        if (lane == 0 && ok) {
            int64_t li = 0;
            for (; i0 + li < i1 && ok; ++li) {
                const int st = (int)(li % kStages);
                ok = mbar_wait(&tready[st], (uint32_t)(li / kStages) & 1, 709);
                if (!ok) break;
                const int64_t i = i0 + li, r = i / a.R;
                const int t = (int)(i % a.R), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
                uint8_t* sb = stages + st * kStageBytes;
                tma_store_3d(&tmap_dq, sb, p * 64, t * kTileTok, b);
                tma_store_3d(&tmap_dnum, sb + kTileBytes, p * 64, t * kTileTok, b);
                bulk_commit_group();
                bulk_wait_group_read<0>();
                mbar_arrive(&empty[st]);
            }
            bulk_wait_group<0>();
        }
    } else {
        // ------------------------------------------------ workers: warp w takes TMEM
        // quadrant w % 4 and head (w / 4) % 2 of the pair, its group alternate tiles
        const int wi = warp - 4;
        const int grp = wi >> 3;
        const int j = (wi >> 2) & 1;
        const int q = warp & 3;
        const int row = 32 * q + lane;
        auto transform = [&](int64_t li, float& rq) -> bool {
            const int st = (int)(li % kStages);
            if (!mbar_wait(&full[st], (uint32_t)(li / kStages) & 1, 710)) return false;
            const int64_t i = i0 + li, r = i / a.R;
            const int t = (int)(i % a.R), p = (int)(r % a.Pp);
            const int h = p * 2 + j;
            const bool live = (t * kTileTok + row < a.N) && h < a.H;
            rq = phi_inplace_sw128<false>(stages + st * kStageBytes, row, j * 4,
                                          sgain + (live ? h : 0) * kD, a.eps, a.norm != 0, !live);
            fence_proxy_async_smem();
            mbar_arrive(&aready[st]);
            return true;
        };
        // epilogue A: dnum (bf16 over the dO tile) and dden
        auto epi_a = [&](int64_t li, float rq, float& dden) -> bool {
            const int st = (int)(li % kStages), tb = (int)(li & 1);
            if (!mbar_wait(&mma1[st], (uint32_t)(li / kStages) & 1, 711)) return false;
            tc_fence_after_sync();
            const int64_t i = i0 + li, r = i / a.R;
            const int t = (int)(i % a.R), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
            const int h = p * 2 + j;
            const int64_t tok = (int64_t)t * kTileTok + row;
            const bool live = tok < a.N && h < a.H;
            const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + tb * kBufCols + j * kNS;
            float dn[2];
            tmem_ld2(ta + p2::kDenHi, dn);
            tmem_wait_ld();
            const float den = rq * (dn[0] + dn[1]);
            const float inv = 1.f / (den + a.eps);
            uint8_t* gtile = stages + st * kStageBytes + kTileBytes;
            float dot = 0.f;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float hi[16], lo[16];
                tmem_ld16(ta + 16 * hf, hi);
                tmem_ld16(ta + p2::kLoRow + 16 * hf, lo);
                tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    uint8_t* gp = gtile + sw128_offset(row, j * 4 + 2 * hf + cc);
                    const uint4 g4 = *reinterpret_cast<const uint4*>(gp);
                    const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
                    float dn8[8];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float go0 = bf16lo(gw[u]), go1 = bf16hi(gw[u]);
                        const float o0 = rq * (hi[8 * cc + 2 * u] + lo[8 * cc + 2 * u]) * inv;
                        const float o1 = rq * (hi[8 * cc + 2 * u + 1] + lo[8 * cc + 2 * u + 1]) * inv;
                        dot = fmaf(go0, o0, fmaf(go1, o1, dot));
                        dn8[2 * u] = go0 * inv;
                        dn8[2 * u + 1] = go1 * inv;
                    }
                    uint4 w;
                    w.x = pack_bf16x2(dn8[0], dn8[1]);
                    w.y = pack_bf16x2(dn8[2], dn8[3]);
                    w.z = pack_bf16x2(dn8[4], dn8[5]);
                    w.w = pack_bf16x2(dn8[6], dn8[7]);
                    if (!live) w = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(gp) = w;
                }
            }
            dden = live ? -dot * inv : 0.f;
            if (live) a.dden[((size_t)b * a.H + h) * a.N + tok] = dden;   // (B, H, N): coalesced
            tc_fence_before_sync();
            fence_proxy_async_smem();
            mbar_arrive(&pready[st]);
            return true;
        };
        // epilogue B: dQ over the Q tile, the gain partial
        auto epi_b = [&](int64_t li, float rq, float dden) -> bool {
            const int st = (int)(li % kStages), tb = (int)(li & 1);
            if (!mbar_wait(&mma2[st], (uint32_t)(li / kStages) & 1, 712)) return false;
            tc_fence_after_sync();
            const int64_t i = i0 + li, r = i / a.R;
            const int t = (int)(i % a.R), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
            const int h = p * 2 + j;
            const int64_t tok = (int64_t)t * kTileTok + row;
            const bool live = tok < a.N && h < a.H;
            const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + tb * kBufCols + j * kNS;
            uint4 qraw[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                             make_uint4(0, 0, 0, 0)};
            if (live) {                                   // requested before the TMEM work
                const uint4* qr = reinterpret_cast<const uint4*>(
                    a.q + ((size_t)b * a.N + tok) * (size_t)(a.H * kD) + (size_t)h * kD);
#pragma unroll
                for (int u = 0; u < 4; ++u) qraw[u] = __ldg(qr + u);
            }
            float dp[kD];
            const float* z = a.s + ((size_t)b * a.H + (h < a.H ? h : 0)) * kStateFloats + kD;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float hi[16], lo[16];
                tmem_ld16(ta + 16 * hf, hi);
                tmem_ld16(ta + kD + 16 * hf, lo);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    dp[16 * hf + u] = (hi[u] + lo[u]) + dden * __ldg(z + (16 * hf + u) * kDP);
            }
            tc_fence_before_sync();
            mbar_arrive(&tfree[tb]);
            phi_bwd_row(dp, qraw, sgain + (h < a.H ? h : 0) * kD, rq, a.norm != 0, live,
                        stages + st * kStageBytes, row, j * 4);
            fence_proxy_async_smem();
            mbar_arrive(&tready[st]);
            if (a.norm) {
                warp_reduce_scatter32(dp, lane);
                a.gpart[((size_t)i * 4 + q) * (2 * kD) + j * kD + lane] = dp[0];
            }
            return true;
        };
        // per group: T(first); then for each of its tiles li: A(li), T(next), B(li)
        int64_t li = grp;
        float r_cur = 1.f, r_next = 1.f, dden = 0.f;
        if (ok && i0 + li < i1) ok = transform(li, r_cur);
        for (; i0 + li < i1 && ok; li += 2) {
            ok = epi_a(li, r_cur, dden);
            if (ok && i0 + li + 2 < i1) ok = transform(li + 2, r_next);
            if (ok) ok = epi_b(li, r_cur, dden);
            r_cur = r_next;
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// dg[c] for c = h D + d (head pair p = h / 2, j = h % 2) = the sum over batch items,
// the row's tiles and the 4 quadrants of gpart[(b Pp + p) R + t][quadrant][j][d]:
// grid (Pp, 32 slices of the tile list), 256 threads = 4 interleaved streams x 64
// channels; each stream adds its entries in order, the streams are added in order
// into slice partials part[p][slice][64], and gain_combine_slices adds the slices in
// order, so the result is reproducible.
constexpr int kGainSlices = 32;

__global__ void __launch_bounds__(256)
gain_combine_tiles(const float* __restrict__ gpart, float* __restrict__ part, int B, int Pp, int R)
{
    __shared__ float acc4[4][2 * kD];
    const int p = blockIdx.x, sl = blockIdx.y, s = threadIdx.x >> 6, ch = threadIdx.x & 63;
    const int per_b = R * 4;                                // (tile, quadrant) entries per batch item
    const int64_t total = (int64_t)B * per_b;
    const int64_t k0 = total * sl / kGainSlices, k1 = total * (sl + 1) / kGainSlices;
    float acc = 0.f;
    int64_t b = k0 / per_b;
    int rem = (int)(k0 % per_b);
    const float* base = gpart + (size_t)p * R * 4 * (2 * kD) + ch;
    const size_t bstride = (size_t)Pp * R * 4 * (2 * kD);
    // entries k0 + s, k0 + s + 4, ... below k1, walked as (b, rem) without divisions
    rem += s;
    while (rem >= per_b) { rem -= per_b; ++b; }
    for (int64_t k = k0 + s; k < k1; k += 4) {
        acc += base[b * bstride + (size_t)rem * (2 * kD)];
        rem += 4;
        while (rem >= per_b) { rem -= per_b; ++b; }
    }
    acc4[s][ch] = acc;
    __syncthreads();
    if (threadIdx.x < 2 * kD)
        part[((size_t)p * kGainSlices + sl) * (2 * kD) + ch] =
            ((acc4[0][ch] + acc4[1][ch]) + acc4[2][ch]) + acc4[3][ch];
}

__global__ void __launch_bounds__(256)
gain_combine_slices(const float* __restrict__ part, float* __restrict__ dg, int Pp, int H)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;   // channel h D + d
    if (c >= H * kD) return;
    const int h = c / kD, p = h / 2, ch = (h % 2) * kD + c % kD;
    float v = 0.f;
    for (int sl = 0; sl < kGainSlices; ++sl) v += part[((size_t)p * kGainSlices + sl) * (2 * kD) + ch];
    dg[c] = v;
}

}  // namespace sana
