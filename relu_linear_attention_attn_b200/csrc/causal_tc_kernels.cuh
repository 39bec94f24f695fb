// The prefix (causal) form of Eq. (1) on the tensor cores.  The explainer page of
// the Sana notes ("线性 DiT") describes linear attention as a cumulative prefix
// sum; token n sees keys j <= n:
//     O_n = phi(Q_n) S_n[:, :D] / (phi(Q_n) S_n[:, D] + eps),
//     S_n = sum_{j <= n} phi(K_j)^T [V_j | 1].
// Chunked over 128 tokens (the UMMA M): for query n of chunk c,
//     S_n = P_c + sum_{j in chunk c, j <= n} phi(K_j)^T [V_j | 1],
// P_c the state of every earlier chunk, so
//     [num_n | den_n] = phi(Q_n) P_c + sum_{j <= n} (phi(Q_n) . phi(K_j)) [V_j | 1].
// Three launches:
//   1. kv_partials_persistent<true>: the state of every chunk (pass 1 with rows of
//      one chunk: up to two partial slots per chunk);
//   2. causal_prefix_states: per (b, h) the exclusive prefix over chunks, summing
//      each chunk's slots in slot order and the chunks in chunk order
//      (reproducible);
//   3. causal_apply_tc: per (b, head pair, chunk), on the tensor cores:
//        U1  P_h = phi(Q_h) phi(K_h)^T            (M = N = 128, K = 32)
//            D_h = phi(Q_h) [P_c hi | lo]          (N = 80, pass 2's operand)
//        the epilogue zeroes P_h[n][j] for j > n and writes it as bf16 (K-major A)
//        U2  D_h[:, 0:48] += P_h [V_h^T ; 1 ; 0]   (N = 48, K = 128)
//            the row of ones adds sum_{j <= n} P_h[n][j] to the normaliser column
//        O = (D[e] + D[48 + e]) / (D[32] + D[33] + eps).
#pragma once

#include "sana_common.cuh"
#include "sm100_primitives.cuh"
#include "tc_kernels.cuh"

namespace sana {

constexpr int kCausalTcChunk = 128;        // tokens per chunk (UMMA M of the apply)

// Exclusive prefix over the chunks of each (b, h): pre[b][h][c] = sum_{c' < c}
// sum_s part[b][h][c'][s] (both [e][d], column e major).  Grid B * H, 264 threads:
// thread t owns the 16 bytes t of a state and walks the chunks in order, loading
// eight chunks ahead.  ns_of(row) gives the slot count of a pass-1 chunk row.
struct PrefixArgs {
    const float* part;   // [B][H][Cc][Smax][D+1][D]
    float* pre;          // [B][H][Cc][D+1][D]
    int H, G, Cc, Smax;
    int64_t R1, T1, P1;  // pass-1 plan (stages per chunk row, items, CTAs)
};

__global__ void __launch_bounds__(kStateFloats / 4)
causal_prefix_states(const PrefixArgs a)
{
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const int i4 = threadIdx.x;
    const float4* src = reinterpret_cast<const float4*>(a.part) + bh * a.Cc * a.Smax * (kStateFloats / 4);
    float4* dst = reinterpret_cast<float4*>(a.pre) + bh * a.Cc * (kStateFloats / 4);
    const int64_t row0 = ((int64_t)b * a.G + h / p1::kGroupHeads) * a.Cc;    // pass-1 row of chunk 0
    float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = 0; c0 < a.Cc; c0 += 8) {
        float4 x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            x[k] = make_float4(0.f, 0.f, 0.f, 0.f);
            const int c = c0 + k;
            if (c < a.Cc) {
                const int ns = p1_row_slots(row0 + c, a.R1, a.T1, a.P1);
                for (int s = 0; s < ns; ++s) {
                    const float4 v = __ldcg(src + ((int64_t)c * a.Smax + s) * (kStateFloats / 4) + i4);
                    x[k].x += v.x; x[k].y += v.y; x[k].z += v.z; x[k].w += v.w;
                }
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int c = c0 + k;
            if (c < a.Cc) {
                dst[(int64_t)c * (kStateFloats / 4) + i4] = run;
                run.x += x[k].x; run.y += x[k].y; run.z += x[k].z; run.w += x[k].w;
            }
        }
    }
}

namespace ca {
constexpr int kTok = kCausalTcChunk;
constexpr int kTile = kTok * 128;                  // 128 tokens x 64 channels (a head pair)
constexpr int kStageBytes = 3 * kTile;             // [Q | K | V]
constexpr int kStages = 2;
constexpr int kVtRows = 48;                        // V^T rows: 32 values, ones, zeros
constexpr int kVtAtom = kVtRows * 128;             // 64 keys of every row
constexpr int kVtHead = 2 * kVtAtom;
constexpr int kPsAtom = kTok * 128;                // 64 keys of every query row
constexpr int kPsHead = 2 * kPsAtom;
constexpr int kBopBytes = p2::kBopBytes;
constexpr int kStagingBytes = 2 * kStateFloats * 4;
constexpr int kPCol = 0;                           // P of head j at 128 j
constexpr int kDCol = 256;                         // D of head j at 256 + 80 j
constexpr int kTmemCols = 512;
constexpr int kGroupThreads = 256;                 // a transform or epilogue group: 8 warps
constexpr int kThreads = 32 * (4 + 16);
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 2 * kVtHead + 2 * kPsHead + 2 * kBopBytes +
                           kStagingBytes + 512;
static_assert(kSmemBytes <= 232448, "shared memory");
}  // namespace ca

struct CaArgs {
    const float* pre;    // [B][H][Cc][D+1][D] prefix states
    const float* gq;     // [C] or nullptr (norm off); 16-byte aligned
    const float* gk;
    int64_t T;           // items: B * Pp rows x Cc chunks
    int N, H, Pp, Cc, P;
    float eps;
    int norm;
};

__global__ void __launch_bounds__(ca::kThreads, 1)
causal_apply_tc(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_o,
                const CaArgs a)
{
    using namespace ca;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* stages = smem;
    uint8_t* vt = stages + kStages * kStageBytes;
    uint8_t* ps = vt + 2 * kVtHead;
    uint8_t* bop = ps + 2 * kPsHead;
    float* staging = (float*)(bop + 2 * kBopBytes);
    uint64_t* full = (uint64_t*)(staging + kStagingBytes / 4);
    uint64_t* sempty = full + kStages;
    uint64_t* aready = sempty + kStages;
    uint64_t* bfull = aready + kStages;
    uint64_t* bempty = bfull + 2;
    uint64_t* pdone = bempty + 2;
    uint64_t* psready = pdone + 1;
    uint64_t* mmadone = psready + 1;
    uint64_t* u2done = mmadone + 1;
    uint64_t* tfree = u2done + 1;
    uint64_t* ofull = tfree + 1;
    uint64_t* sready = ofull + 1;
    uint64_t* drain = sready + 1;
    uint32_t* tmem_slot = (uint32_t*)(drain + 1);

    const int64_t cta = blockIdx.x;
    const int64_t i0 = range_begin(cta, a.T, a.P), i1 = range_begin(cta + 1, a.T, a.P);
    const int64_t n = i1 - i0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&sempty[i], 1);
            mbar_init(&aready[i], kGroupThreads);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bfull[i], 32);
            mbar_init(&bempty[i], 1);
        }
        mbar_init(pdone, 1);
        mbar_init(psready, kGroupThreads);
        mbar_init(mmadone, 1);
        mbar_init(u2done, 1);
        mbar_init(tfree, kGroupThreads);
        mbar_init(ofull, kGroupThreads);
        mbar_init(sready, 1);
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
        prefetch_tmap(&tmap_o);
    }
    // constant parts of the operands: rows 34..47 of both B-operand buffers, and
    // rows 32 (ones: the normaliser's intra-chunk sum) and 33..47 (zeros) of V^T
    for (int i = threadIdx.x; i < 2 * (p2::kLoRow - p2::kDenLo - 1) * 8; i += blockDim.x) {
        const int rb = i / ((p2::kLoRow - p2::kDenLo - 1) * 8), rem = i % ((p2::kLoRow - p2::kDenLo - 1) * 8);
        *reinterpret_cast<uint4*>(bop + rb * kBopBytes + (p2::kDenLo + 1 + rem / 8) * 128 +
                                  (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
    }
    for (int i = threadIdx.x; i < 2 * 2 * 16 * 8; i += blockDim.x) {   // [head][atom][row 32..47][chunk]
        const int hh = i / (2 * 16 * 8), at = (i / (16 * 8)) % 2, rw = 32 + (i / 8) % 16, ch = i % 8;
        const uint32_t one2 = 0x3F803F80u;                             // two bf16 ones
        const uint32_t w = rw == 32 ? one2 : 0u;
        *reinterpret_cast<uint4*>(vt + hh * kVtHead + at * kVtAtom + sw128_offset(rw, ch)) =
            make_uint4(w, w, w, w);
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
    bool ok = n > 0;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer: Q, K, V tiles
        if (lane == 0 && ok) {
            int64_t last = -1;
            for (int64_t li = 0; li < n; ++li) {
                const int s = (int)(li & 1);
                if (li >= kStages) ok = mbar_wait(&sempty[s], (uint32_t)((li >> 1) - 1) & 1, 901);
                if (!ok) break;
                const int64_t i = i0 + li, r = i / a.Cc;
                const int c = (int)(i % a.Cc), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
                uint8_t* sb = stages + s * kStageBytes;
                mbar_arrive_expect_tx(&full[s], kStageBytes);
                tma_load_3d(sb, &tmap_q, &full[s], p * 64, c * kTok, b);
                tma_load_3d(sb + kTile, &tmap_k, &full[s], p * 64, c * kTok, b);
                tma_load_3d(sb + 2 * kTile, &tmap_v, &full[s], p * 64, c * kTok, b);
                last = li;
            }
            if (!ok) {
                for (int s = 0; s < kStages; ++s) {
                    const int64_t lj = last - ((last - s) % kStages + kStages) % kStages;
                    if (last >= 0 && lj >= 0)
                        mbar_wait(&full[s], (uint32_t)(lj >> 1) & 1, 902);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer (one elected lane)
        if (ok) {
            const uint32_t idesc_p = make_idesc_bf16(128, 128, false, false);
            const uint32_t idesc_d = make_idesc_bf16(128, p2::kN, false, false);
            const uint32_t idesc_v = make_idesc_bf16(128, kVtRows, false, false);
            const uint64_t st0 = make_smem_desc(smem_u32(stages), 16, 1024, kSwizzle128B);
            const uint64_t bo0 = make_smem_desc(smem_u32(bop), 16, 1024, kSwizzle128B);
            const uint64_t ps0 = make_smem_desc(smem_u32(ps), 16, 1024, kSwizzle128B);
            const uint64_t vt0 = make_smem_desc(smem_u32(vt), 16, 1024, kSwizzle128B);
            for (int64_t li = 0; li < n; ++li) {
                const int s = (int)(li & 1), rb = (int)(li & 1);
                if (lane == 0) {
                    ok = mbar_wait(&aready[s], (uint32_t)(li >> 1) & 1, 903);
                    if (ok) ok = mbar_wait(&bfull[rb], (uint32_t)(li >> 1) & 1, 904);
                    if (ok && li >= 1) ok = mbar_wait(tfree, (uint32_t)(li - 1) & 1, 905);
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after_sync();
                const uint64_t qd = st0 + (uint64_t)((s * kStageBytes) >> 4);
                const uint64_t kd = qd + (uint64_t)(kTile >> 4);
                const uint64_t bd = bo0 + (uint64_t)((rb * kBopBytes) >> 4);
#pragma unroll
                for (int jh = 0; jh < 2; ++jh) {
                    const uint32_t dp = tmem + kPCol + 128 * jh, dd = tmem + kDCol + p2::kN * jh;
                    umma_bf16_elect(dp, qd + 4 * jh, kd + 4 * jh, idesc_p, false);
                    umma_bf16_elect(dp, qd + 4 * jh + 2, kd + 4 * jh + 2, idesc_p, true);
                    umma_bf16_elect(dd, qd + 4 * jh, bd + 4 * jh, idesc_d, false);
                    umma_bf16_elect(dd, qd + 4 * jh + 2, bd + 4 * jh + 2, idesc_d, true);
                }
                umma_commit_elect(pdone);
                umma_commit_elect(&bempty[rb]);
                if (lane == 0) ok = mbar_wait(psready, (uint32_t)li & 1, 906);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after_sync();
#pragma unroll
                for (int jh = 0; jh < 2; ++jh) {
                    const uint32_t dd = tmem + kDCol + p2::kN * jh;
#pragma unroll
                    for (int k = 0; k < kTok / 16; ++k) {
                        const uint64_t off_p = (uint64_t)((jh * kPsHead + (k >> 2) * kPsAtom) >> 4) + 2 * (k & 3);
                        const uint64_t off_v = (uint64_t)((jh * kVtHead + (k >> 2) * kVtAtom) >> 4) + 2 * (k & 3);
                        umma_bf16_elect(dd, ps0 + off_p, vt0 + off_v, idesc_v, true);
                    }
                }
                umma_commit_elect(mmadone);
                umma_commit_elect(u2done);
            }
            umma_commit_elect(drain);
            if (lane == 0) mbar_wait(drain, 0, 907);
            __syncwarp();
        }
    } else if (warp == 2) {
        // ------------------------------------------------ B operand of each chunk's
        // prefix state (the pair's two heads), as pass 2 builds it from a state
        int64_t li = 0;
        for (; li < n && ok; ++li) {
            const int rb = (int)(li & 1);
            if (li >= 2) ok = mbar_wait(&bempty[rb], (uint32_t)((li >> 1) - 1) & 1, 908);
            if (!ok) break;
            const int64_t i = i0 + li, r = i / a.Cc;
            const int c = (int)(i % a.Cc), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
            const int h0 = 2 * p, nh = min(2, a.H - h0);
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_expect_tx(sready, (uint32_t)(nh * kStateFloats * 4));
                for (int j = 0; j < nh; ++j)
                    bulk_load(staging + j * kStateFloats,
                              a.pre + (((size_t)b * a.H + h0 + j) * a.Cc + c) * kStateFloats,
                              kStateFloats * 4, sready);
            }
            ok = mbar_wait(sready, (uint32_t)li & 1, 909);
            if (!ok) break;
            uint8_t* dst = bop + rb * kBopBytes;
            const int d0 = lane & ~1;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int chunk = j * 4 + d0 / 8, off = (d0 % 8) * 2;
#pragma unroll
                for (int e = 0; e < kDP; ++e) {
                    const float x = j < nh ? staging[j * kStateFloats + e * kD + lane] : 0.f;
                    const float xp = __shfl_xor_sync(0xffffffffu, x, 1);
                    const float xe = (lane & 1) ? xp : x, xo = (lane & 1) ? x : xp;
                    const float he = __bfloat162float(__float2bfloat16_rn(xe));
                    const float ho = __bfloat162float(__float2bfloat16_rn(xo));
                    const int row = (lane & 1) ? (e < kD ? p2::kLoRow + e : p2::kDenLo) : e;
                    const uint32_t w = (lane & 1) ? pack_bf16x2(xe - he, xo - ho) : pack_bf16x2(he, ho);
                    *reinterpret_cast<uint32_t*>(dst + sw128_offset(row, chunk) + off) = w;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            mbar_arrive(&bfull[rb]);
        }
    } else if (warp == 3) {
        // ------------------------------------------------ O stores (over the Q tile)
        if (lane == 0 && ok) {
            for (int64_t li = 0; li < n && ok; ++li) {
                const int s = (int)(li & 1);
                ok = mbar_wait(ofull, (uint32_t)li & 1, 910);
                if (!ok) break;
                const int64_t i = i0 + li, r = i / a.Cc;
                const int c = (int)(i % a.Cc), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
                tma_store_3d(&tmap_o, stages + s * kStageBytes, p * 64, c * kTok, b);
                bulk_commit_group();
                bulk_wait_group_read<0>();
                mbar_arrive(&sempty[s]);
            }
            bulk_wait_group<0>();
        }
    } else if (warp < 12) {
        // ------------------------------------------------ phi(Q), phi(K) in place, V^T:
        // warp w takes token row 32 (w % 4) + lane of the chunk, head (w - 4) / 4 of
        // the pair
        // (the gains are read from global memory, 16-byte aligned: checked on the host)
        const int tw = warp - 4, jh = tw >> 2, row = 32 * (tw & 3) + lane;
        for (int64_t li = 0; li < n && ok; ++li) {
            const int s = (int)(li & 1);
            const int64_t i = i0 + li, r = i / a.Cc;
            const int c = (int)(i % a.Cc), p = (int)(r % a.Pp);
            ok = mbar_wait(&full[s], (uint32_t)(li >> 1) & 1, 911);
            if (!ok) break;
            const int h = 2 * p + jh;
            const bool live = (c * kTok + row < a.N) && h < a.H;
            const int hg = live ? h : 0;
            uint8_t* sb = stages + s * kStageBytes;
            phi_inplace_sw128<true>(sb, row, jh * 4, a.norm ? a.gq + hg * kD : nullptr, a.eps,
                                    a.norm != 0, !live);
            phi_inplace_sw128<true>(sb + kTile, row, jh * 4, a.norm ? a.gk + hg * kD : nullptr, a.eps,
                                    a.norm != 0, !live);
            // V^T of this head: column `row` (key j = row) of rows e = 0..31
            if (li >= 1) ok = mbar_wait(u2done, (uint32_t)(li - 1) & 1, 912);
            if (!ok) break;
            uint4 u[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
                u[cc] = *reinterpret_cast<const uint4*>(sb + 2 * kTile + sw128_offset(row, jh * 4 + cc));
            uint8_t* vh = vt + jh * kVtHead + (row >> 6) * kVtAtom;
            const int kch = (row & 63) >> 3, kb = (row & 7) * 2;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const uint32_t wds[4] = {u[cc].x, u[cc].y, u[cc].z, u[cc].w};
#pragma unroll
                for (int k2 = 0; k2 < 4; ++k2) {
                    const int e = cc * 8 + k2 * 2;
                    *reinterpret_cast<uint16_t*>(vh + sw128_offset(e, kch) + kb) = (uint16_t)(wds[k2] & 0xffffu);
                    *reinterpret_cast<uint16_t*>(vh + sw128_offset(e + 1, kch) + kb) = (uint16_t)(wds[k2] >> 16);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&aready[s]);
        }
    } else {
        // ------------------------------------------------ epilogues: warp w reads TMEM lane
        // quadrant w % 4 (query row n = 32 (w % 4) + lane), head (w - 12) / 4 of the pair
        const int ew = warp - 12, jh = ew >> 2, q = warp & 3, nrow = 32 * q + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        for (int64_t li = 0; li < n && ok; ++li) {
            const int s = (int)(li & 1);
            ok = mbar_wait(pdone, (uint32_t)li & 1, 913);
            if (ok && li >= 1) ok = mbar_wait(u2done, (uint32_t)(li - 1) & 1, 914);
            if (!ok) break;
            tc_fence_after_sync();
            // P_h[n][j] for j <= n, as bf16 into the K-major A operand of U2
            uint8_t* ph = ps + jh * kPsHead;
#pragma unroll 1
            for (int kc = 0; kc < kTok / 32; ++kc) {
                float v[32];
                tmem_ld16(lane_base + kPCol + 128 * jh + 32 * kc, v);
                tmem_ld16(lane_base + kPCol + 128 * jh + 32 * kc + 16, v + 16);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (32 * kc + i > nrow) v[i] = 0.f;
                uint8_t* at = ph + (kc >> 1) * kPsAtom;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 w;
                    w.x = pack_bf16x2(v[8 * cc + 0], v[8 * cc + 1]);
                    w.y = pack_bf16x2(v[8 * cc + 2], v[8 * cc + 3]);
                    w.z = pack_bf16x2(v[8 * cc + 4], v[8 * cc + 5]);
                    w.w = pack_bf16x2(v[8 * cc + 6], v[8 * cc + 7]);
                    *reinterpret_cast<uint4*>(at + sw128_offset(nrow, (kc & 1) * 4 + cc)) = w;
                }
            }
            tc_fence_before_sync();
            fence_proxy_async_smem();
            mbar_arrive(psready);
            // O = (hi + lo) / (den_hi + den_lo + eps), over the Q tile of the stage
            ok = mbar_wait(mmadone, (uint32_t)li & 1, 915);
            if (!ok) break;
            tc_fence_after_sync();
            const uint32_t ta = lane_base + kDCol + p2::kN * jh;
            float hi[kD + 2], lo[kD];
            tmem_ld16(ta, hi);
            tmem_ld16(ta + 16, hi + 16);
            tmem_ld2(ta + p2::kDenHi, hi + kD);
            tmem_ld16(ta + p2::kLoRow, lo);
            tmem_ld16(ta + p2::kLoRow + 16, lo + 16);
            tmem_wait_ld();
            const float inv = __frcp_rn((hi[kD] + hi[kD + 1]) + a.eps);
            uint8_t* ot = stages + s * kStageBytes;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float o[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) o[u] = (hi[8 * cc + u] + lo[8 * cc + u]) * inv;
                uint4 w;
                w.x = pack_bf16x2(o[0], o[1]);
                w.y = pack_bf16x2(o[2], o[3]);
                w.z = pack_bf16x2(o[4], o[5]);
                w.w = pack_bf16x2(o[6], o[7]);
                *reinterpret_cast<uint4*>(ot + sw128_offset(nrow, jh * 4 + cc)) = w;
            }
            tc_fence_before_sync();
            fence_proxy_async_smem();
            mbar_arrive(tfree);
            mbar_arrive(ofull);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace sana
