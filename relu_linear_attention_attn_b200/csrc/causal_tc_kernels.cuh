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
//   3. causal_apply_tc: per (b, head pair, chunk), head by head, on the tensor cores:
//        U1  P_h = phi(Q_h) phi(K_h)^T            (M = N = 128, K = 32)
//        the epilogue zeroes P_h[n][j] for j > n, writes it as bf16 (K-major A) and
//        sums each masked row in fp32 (the chunk's own normaliser share)
//        U2  D_h = phi(Q_h) [P_c hi | lo]          (N = 80, pass 2's operand)
//            D_h[:, 0:32] += P_h V_h                (N = 32, K = 128, V MN-major)
//        O = (D[e] + D[48 + e]) / (D[32] + D[33] + row sum + eps).
#pragma once

#include "sana_common.cuh"
#include "sm100_primitives.cuh"
#include "tc_kernels.cuh"

namespace sana {

constexpr int kCausalTcChunk = 128;        // tokens per chunk (UMMA M of the apply)

// Exclusive prefix over the chunks of each (b, h): pre[b][h][c] = sum_{c' < c}
// sum_s part[b][h][c'][s] (both [e][d], column e major).  Grid B * H, 264 threads:
// thread t owns the 16 bytes t of a state and walks the chunks in order, loading
// eight chunks ahead; each chunk's slots are summed in slot order and the chunks in
// chunk order, so the result is reproducible.
struct PrefixArgs {
    const float* part;   // [B][H][Cc][Smax][D+1][D]
    float* pre;          // [B][H][Cc][D+1][D]
    int H, G, Cc, Smax;
    int64_t R1, T1, P1;  // pass-1 plan (stages per chunk row, items, CTAs)
};

constexpr int kPrefixThreads = kStateFloats / 4;

__global__ void __launch_bounds__(kPrefixThreads)
causal_prefix_states(const PrefixArgs a)
{
    constexpr int kBatch = 8;                      // chunks whose loads are in flight at once
    constexpr int kSplitWords = 1024;              // chunks whose slot counts fit the bit table
    __shared__ uint32_t split[kSplitWords];        // bit c: chunk c has two pass-1 slots
    pdl_launch_dependents();                       // the apply reads `pre` only after its own wait
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const int i4 = threadIdx.x;
    const float4* src = reinterpret_cast<const float4*>(a.part) + bh * a.Cc * a.Smax * (kStateFloats / 4);
    float4* dst = reinterpret_cast<float4*>(a.pre) + bh * a.Cc * (kStateFloats / 4);
    const int64_t row0 = ((int64_t)b * a.G + h / p1::kGroupHeads) * a.Cc;    // pass-1 row of chunk 0
    // With two pass-1 items per chunk, a chunk has two slots exactly when a pass-1 CTA's
    // range starts at its second item: one division per CTA boundary instead of two per
    // chunk and thread.
    const bool table = a.R1 == 2 && a.Cc <= kSplitWords * 32;
    if (table) {
        for (int w = threadIdx.x; w < (a.Cc + 31) / 32; w += blockDim.x) split[w] = 0u;
        __syncthreads();
        for (int64_t c = 1 + threadIdx.x; c < a.P1; c += blockDim.x) {
            const int64_t bnd = range_begin(c, a.T1, a.P1);
            const int64_t cr = (bnd >> 1) - row0;
            if ((bnd & 1) && cr >= 0 && cr < a.Cc) atomicOr(&split[cr >> 5], 1u << (cr & 31));
        }
        __syncthreads();
    }
    // Slot 0 of every chunk and slot 1 where it exists are loaded for a whole batch of
    // chunks before any is summed (straight-line predicated loads: a run-time slot
    // loop would leave one round trip per chunk); chunks with more than two slots
    // (never produced by the chunked pass 1) take the general loop.
    float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = 0; c0 < a.Cc; c0 += kBatch) {
        float4 v0[kBatch], v1[kBatch];
        int nsk[kBatch];
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const int c = c0 + k;
            nsk[k] = c < a.Cc ? (table ? 1 + (int)((split[c >> 5] >> (c & 31)) & 1u)
                                       : p1_row_slots(row0 + c, a.R1, a.T1, a.P1))
                              : 0;
        }
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const float4* sc = src + (int64_t)(c0 + k) * a.Smax * (kStateFloats / 4) + i4;
            v0[k] = nsk[k] > 0 ? __ldcg(sc) : make_float4(0.f, 0.f, 0.f, 0.f);
            v1[k] = nsk[k] > 1 ? __ldcg(sc + kStateFloats / 4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            if (nsk[k] == 0) continue;
            const int c = c0 + k;
            float4 x = v0[k];                              // slot order: 0, 1, then the rest
            if (nsk[k] > 1) { x.x += v1[k].x; x.y += v1[k].y; x.z += v1[k].z; x.w += v1[k].w; }
            for (int s = 2; s < nsk[k]; ++s) {
                const float4 v = __ldcg(src + ((int64_t)c * a.Smax + s) * (kStateFloats / 4) + i4);
                x.x += v.x; x.y += v.y; x.z += v.z; x.w += v.w;
            }
            dst[(int64_t)c * (kStateFloats / 4) + i4] = run;
            run.x += x.x; run.y += x.y; run.z += x.z; run.w += x.w;
        }
    }
}

namespace ca {
constexpr int kTok = kCausalTcChunk;
constexpr int kTile = kTok * 128;                  // 128 tokens x 64 channels (a head pair)
constexpr int kQSlots = 3;                         // Q tiles (phi(Q) in place, then O over it)
constexpr int kKSlots = 2;                         // K tiles (phi(K) in place)
constexpr int kVSlots = 3;                         // V tiles (the MN-major B operand of U2)
constexpr int kPsAtom = kTok * 128;                // 64 keys of every query row
constexpr int kPsBuf = 2 * kPsAtom;                // one head's masked P, bf16
constexpr int kBopBytes = p2::kBopBytes;
constexpr int kBufCols = 128;                      // TMEM per sub-item: P, then D over it
constexpr int kTmemBufs = 4;
constexpr int kTmemCols = kTmemBufs * kBufCols;
constexpr int kGroupThreads = 256;                 // the transform or the epilogue warps
constexpr int kThreads = 32 * (4 + 16);
constexpr int kRowSumBytes = kTmemBufs * 2 * kTok * 4;   // [sub-item % 4][key half][query row]
constexpr int kPrePer = (2 * kDP * (kD / 2) + kGroupThreads - 1) / kGroupThreads;   // B items per thread
constexpr int kSmemBytes = 1024 + (kQSlots + kKSlots + kVSlots) * kTile + 2 * kPsBuf + 2 * kBopBytes +
                           kRowSumBytes + 512;
static_assert(kSmemBytes <= 232448, "shared memory");
static_assert(kTmemCols <= 512, "TMEM");
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

// Work item li = (b, head pair p, chunk c); sub-item u = 2 li + j is head j of the
// pair.  Per sub-item, on the tensor cores:
//   U1(u)  P = phi(Q_j) phi(K_j)^T                      -> TMEM buffer u % 4
//   A(u)   epilogue: P masked to keys j <= n, bf16      -> P_s[u % 2] (K-major A);
//          the row sums of the masked values (the chunk's own share of the
//          normaliser, summed before the bf16 rounding) go to shared memory
//   U2(u)  D = phi(Q_j) [P_c hi | lo] + P_s V_j          -> the same TMEM buffer
//          (V_j straight from its landing tile, as an MN-major B operand)
//   B(u)   epilogue: O = (D[e] + D[48 + e]) / (D[32] + D[33] + row sum + eps), over
//          the Q tile
// The issuer runs U1(u + 1) before U2(u) and the epilogue warps run A(u) before
// B(u - 1), so the tensor cores work on one sub-item while the epilogue warps work
// on its neighbours.  K tiles leave their ring once both heads' P are formed, V
// tiles once both heads' U2 are done, Q tiles (then O) once their store has read
// them.  The transform warps also build each item's prefix operand, its loads
// issued one item ahead.
__global__ void __launch_bounds__(ca::kThreads, 1)
causal_apply_tc(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_o,
                const CaArgs a)
{
    using namespace ca;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* qring = smem;
    uint8_t* kring = qring + kQSlots * kTile;
    uint8_t* vring = kring + kKSlots * kTile;
    uint8_t* ps = vring + kVSlots * kTile;
    uint8_t* bop = ps + 2 * kPsBuf;
    float* rowsum = (float*)(bop + 2 * kBopBytes);
    uint64_t* qfull = (uint64_t*)((uint8_t*)rowsum + kRowSumBytes);
    uint64_t* qempty = qfull + kQSlots;
    uint64_t* ofull = qempty + kQSlots;
    uint64_t* vfull = ofull + kQSlots;
    uint64_t* vempty = vfull + kVSlots;
    uint64_t* kfull = vempty + kVSlots;
    uint64_t* kempty = kfull + kKSlots;
    uint64_t* qkready = kempty + kKSlots;          // 2
    uint64_t* bfull = qkready + 2;                 // 2
    uint64_t* bempty = bfull + 2;                  // 2
    uint64_t* pdone = bempty + 2;                  // kTmemBufs
    uint64_t* mmadone = pdone + kTmemBufs;         // kTmemBufs
    uint64_t* tfree = mmadone + kTmemBufs;         // kTmemBufs
    uint64_t* psready = tfree + kTmemBufs;         // 2
    uint64_t* u2done = psready + 2;                // 2
    uint64_t* drain = u2done + 2;
    uint32_t* tmem_slot = (uint32_t*)(drain + 1);

    const int64_t cta = blockIdx.x;
    const int64_t i0 = range_begin(cta, a.T, a.P), i1 = range_begin(cta + 1, a.T, a.P);
    const int64_t n = i1 - i0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kQSlots; ++i) {
            mbar_init(&qfull[i], 1);
            mbar_init(&qempty[i], 1);
            mbar_init(&ofull[i], 2 * kGroupThreads);
        }
        for (int i = 0; i < kVSlots; ++i) {
            mbar_init(&vfull[i], 1);
            mbar_init(&vempty[i], 1);
        }
        for (int i = 0; i < kKSlots; ++i) {
            mbar_init(&kfull[i], 1);
            mbar_init(&kempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qkready[i], kGroupThreads);
            mbar_init(&bfull[i], kGroupThreads);
            mbar_init(&bempty[i], 1);
            mbar_init(&psready[i], kGroupThreads);
            mbar_init(&u2done[i], 1);
        }
        for (int i = 0; i < kTmemBufs; ++i) {
            mbar_init(&pdone[i], 1);
            mbar_init(&mmadone[i], 1);
            mbar_init(&tfree[i], kGroupThreads);
        }
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
        prefetch_tmap(&tmap_o);
    }
    // Constant parts of the operands: rows 34..47 of both B-operand buffers, and all
    // of P_s (the blocks of keys after a query's 32-row quadrant are never written).
    for (int i = threadIdx.x; i < 2 * (p2::kLoRow - p2::kDenLo - 1) * 8; i += blockDim.x) {
        const int rb = i / ((p2::kLoRow - p2::kDenLo - 1) * 8), rem = i % ((p2::kLoRow - p2::kDenLo - 1) * 8);
        *reinterpret_cast<uint4*>(bop + rb * kBopBytes + (p2::kDenLo + 1 + rem / 8) * 128 +
                                  (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
    }
    for (int i = threadIdx.x; i < 2 * kPsBuf / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(ps)[i] = make_uint4(0, 0, 0, 0);
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
        // ------------------------------------------------ TMA producer: Q, K, V of each item
        if (lane == 0 && ok) {
            int64_t last = -1;
            for (int64_t li = 0; li < n; ++li) {
                const int qs = (int)(li % kQSlots), ks = (int)(li % kKSlots), vs = (int)(li % kVSlots);
                const int64_t i = i0 + li, r = i / a.Cc;
                const int c = (int)(i % a.Cc), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
                if (li >= kQSlots) ok = mbar_wait(&qempty[qs], (uint32_t)((li / kQSlots) - 1) & 1, 901);
                if (ok && li >= kKSlots) ok = mbar_wait(&kempty[ks], (uint32_t)((li / kKSlots) - 1) & 1, 902);
                if (ok && li >= kVSlots) ok = mbar_wait(&vempty[vs], (uint32_t)((li / kVSlots) - 1) & 1, 903);
                if (!ok) break;
                mbar_arrive_expect_tx(&qfull[qs], kTile);
                tma_load_3d(qring + qs * kTile, &tmap_q, &qfull[qs], p * 64, c * kTok, b);
                mbar_arrive_expect_tx(&kfull[ks], kTile);
                tma_load_3d(kring + ks * kTile, &tmap_k, &kfull[ks], p * 64, c * kTok, b);
                mbar_arrive_expect_tx(&vfull[vs], kTile);
                tma_load_3d(vring + vs * kTile, &tmap_v, &vfull[vs], p * 64, c * kTok, b);
                last = li;
            }
            if (!ok) {   // let every issued copy land before the CTA can exit
                for (int64_t lj = last - (kQSlots - 1) > 0 ? last - (kQSlots - 1) : 0; lj <= last; ++lj)
                    mbar_wait(&qfull[lj % kQSlots], (uint32_t)(lj / kQSlots) & 1, 904);
                for (int64_t lj = last - (kKSlots - 1) > 0 ? last - (kKSlots - 1) : 0; lj <= last; ++lj)
                    mbar_wait(&kfull[lj % kKSlots], (uint32_t)(lj / kKSlots) & 1, 904);
                for (int64_t lj = last - (kVSlots - 1) > 0 ? last - (kVSlots - 1) : 0; lj <= last; ++lj)
                    mbar_wait(&vfull[lj % kVSlots], (uint32_t)(lj / kVSlots) & 1, 904);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer (lane 0 alone, no
        // warp-collective steps between the UMMAs); order U1(0), then per sub-item u:
        // U1(u + 1), U2(u)
        if (ok && lane == 0) {
            const uint32_t idesc_p = make_idesc_bf16(128, 128, false, false);
            const uint32_t idesc_d = make_idesc_bf16(128, p2::kN, false, false);
            const uint32_t idesc_v = make_idesc_bf16(128, kD, false, true);     // V MN-major
            const uint64_t q0 = make_smem_desc(smem_u32(qring), 16, 1024, kSwizzle128B);
            const uint64_t k0 = make_smem_desc(smem_u32(kring), 16, 1024, kSwizzle128B);
            const uint64_t v0 = make_smem_desc(smem_u32(vring), kTile, 1024, kSwizzle128B);
            const uint64_t bo0 = make_smem_desc(smem_u32(bop), 16, 1024, kSwizzle128B);
            const uint64_t ps0 = make_smem_desc(smem_u32(ps), 16, 1024, kSwizzle128B);
            const int64_t nsub = 2 * n;
            auto u1 = [&](int64_t u) -> bool {
                const int64_t li = u >> 1;
                const int j = (int)(u & 1), tb = (int)(u % kTmemBufs);
                if (j == 0 && !mbar_wait(&qkready[li & 1], (uint32_t)(li >> 1) & 1, 905)) return false;
                if (u >= kTmemBufs && !mbar_wait(&tfree[tb], (uint32_t)((u / kTmemBufs) - 1) & 1, 906))
                    return false;
                tc_fence_after_sync();
                const uint64_t qd = q0 + (uint64_t)(((li % kQSlots) * kTile) >> 4) + 4 * j;
                const uint64_t kd = k0 + (uint64_t)(((li % kKSlots) * kTile) >> 4) + 4 * j;
                const uint32_t dp = tmem + tb * kBufCols;
                umma_bf16(dp, qd, kd, idesc_p, false);
                umma_bf16(dp, qd + 2, kd + 2, idesc_p, true);
                umma_commit(&pdone[tb]);
                if (j == 1) umma_commit(&kempty[li % kKSlots]);         // phi(K) read by both heads
                return true;
            };
            auto u2 = [&](int64_t u) -> bool {
                const int64_t li = u >> 1;
                const int j = (int)(u & 1), tb = (int)(u % kTmemBufs), pb = (int)(u & 1);
                const int vs = (int)(li % kVSlots);
                if (!mbar_wait(&psready[pb], (uint32_t)(u >> 1) & 1, 907)) return false;
                if (j == 0 && !mbar_wait(&vfull[vs], (uint32_t)(li / kVSlots) & 1, 908)) return false;
                if (j == 0 && !mbar_wait(&bfull[li & 1], (uint32_t)(li >> 1) & 1, 909)) return false;
                tc_fence_after_sync();
                const uint64_t qd = q0 + (uint64_t)(((li % kQSlots) * kTile) >> 4) + 4 * j;
                const uint64_t bd = bo0 + (uint64_t)(((li & 1) * kBopBytes) >> 4) + 4 * j;
                const uint32_t dd = tmem + tb * kBufCols;
                umma_bf16(dd, qd, bd, idesc_d, false);
                umma_bf16(dd, qd + 2, bd + 2, idesc_d, true);
                // intra-chunk part: A = P_s (K-major, 64 keys per atom), B = V_j (MN-major:
                // head j's 32 channels of each key row; 16 keys = 2048 bytes a step)
                const uint64_t pa = ps0 + (uint64_t)((pb * kPsBuf) >> 4);
                const uint64_t vb = v0 + (uint64_t)((vs * kTile) >> 4) + 4 * j;
#pragma unroll
                for (int k = 0; k < kTok / 16; ++k) {
                    const uint64_t atp = (uint64_t)(((k >> 2) * kPsAtom) >> 4) + 2 * (k & 3);
                    umma_bf16(dd, pa + atp, vb + (uint64_t)k * 128, idesc_v, true);
                }
                umma_commit(&mmadone[tb]);
                umma_commit(&u2done[pb]);
                if (j == 1) {
                    umma_commit(&vempty[vs]);
                    umma_commit(&bempty[li & 1]);
                }
                return true;
            };
            ok = u1(0);
            for (int64_t u = 0; u < nsub && ok; ++u) {
                if (u + 1 < nsub) ok = u1(u + 1);
                if (ok) ok = u2(u);
            }
            umma_commit(drain);
            mbar_wait(drain, 0, 910);
        }
        __syncwarp();
    } else if (warp == 3) {
        // ------------------------------------------------ O stores (over the Q tile)
        if (lane == 0 && ok) {
            for (int64_t li = 0; li < n && ok; ++li) {
                const int qs = (int)(li % kQSlots);
                ok = mbar_wait(&ofull[qs], (uint32_t)(li / kQSlots) & 1, 912);
                if (!ok) break;
                const int64_t i = i0 + li, r = i / a.Cc;
                const int c = (int)(i % a.Cc), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
                tma_store_3d(&tmap_o, qring + qs * kTile, p * 64, c * kTok, b);
                bulk_commit_group();
                bulk_wait_group_read<0>();
                mbar_arrive(&qempty[qs]);
            }
            bulk_wait_group<0>();
        }
    } else if (warp >= 4 && warp < 12) {
        // ------------------------------------------------ phi(Q), phi(K) in place; then the
        // item's prefix operand.  Warp w takes token row 32 (w % 4) + lane of the chunk,
        // head (w - 4) / 4 of the pair (the gains are read from global memory, 16-byte
        // aligned: checked on the host).  For the operand, thread t takes the items
        // (j, e, dp) = t + 256 k: S_j[e][2dp], S_j[e][2dp + 1] of the chunk's prefix.
        const int t = threadIdx.x - 128, tw = warp - 4, jh = tw >> 2, row = 32 * (tw & 3) + lane;
        float2 pv[kPrePer];
        auto load_pre = [&](int64_t li) {
            const int64_t i = i0 + li, r = i / a.Cc;
            const int c = (int)(i % a.Cc), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
            const int nh = min(2, a.H - 2 * p);
#pragma unroll
            for (int k = 0; k < kPrePer; ++k) {
                const int it = t + k * kGroupThreads;
                const int dp = it % (kD / 2), e = (it / (kD / 2)) % kDP, jj = it / (kD / 2 * kDP);
                pv[k] = make_float2(0.f, 0.f);
                if (it < 2 * kDP * (kD / 2) && jj < nh)
                    pv[k] = __ldcg(reinterpret_cast<const float2*>(
                        a.pre + (((size_t)b * a.H + 2 * p + jj) * a.Cc + c) * kStateFloats + e * kD + 2 * dp));
            }
        };
        for (int64_t li = 0; li < n && ok; ++li) {
            const int qs = (int)(li % kQSlots), ks = (int)(li % kKSlots);
            const int64_t i = i0 + li, r = i / a.Cc;
            const int c = (int)(i % a.Cc), p = (int)(r % a.Pp);
            ok = mbar_wait(&qfull[qs], (uint32_t)(li / kQSlots) & 1, 913);
            if (ok) ok = mbar_wait(&kfull[ks], (uint32_t)(li / kKSlots) & 1, 914);
            if (!ok) break;
            const int h = 2 * p + jh;
            const bool live = (c * kTok + row < a.N) && h < a.H;
            const int hg = live ? h : 0;
            phi_inplace_sw128<true>(qring + qs * kTile, row, jh * 4, a.norm ? a.gq + hg * kD : nullptr,
                                    a.eps, a.norm != 0, !live);
            phi_inplace_sw128<true>(kring + ks * kTile, row, jh * 4, a.norm ? a.gk + hg * kD : nullptr,
                                    a.eps, a.norm != 0, !live);
            fence_proxy_async_smem();
            mbar_arrive(&qkready[li & 1]);
            // the prefix operand, hi / lo bf16 as pass 2 builds it
            if (li == 0) {
                pdl_wait_primary();                               // the states come from the prefix kernel
                load_pre(0);
            }
            if (li >= 2) ok = mbar_wait(&bempty[li & 1], (uint32_t)((li >> 1) - 1) & 1, 915);
            if (!ok) break;
            uint8_t* dst = bop + (li & 1) * kBopBytes;
#pragma unroll
            for (int k = 0; k < kPrePer; ++k) {
                const int it = t + k * kGroupThreads;
                if (it >= 2 * kDP * (kD / 2)) continue;
                const int dp = it % (kD / 2), e = (it / (kD / 2)) % kDP, jj = it / (kD / 2 * kDP);
                const int d0 = 2 * dp;
                const float h0 = __bfloat162float(__float2bfloat16_rn(pv[k].x));
                const float h1 = __bfloat162float(__float2bfloat16_rn(pv[k].y));
                const int chunk = jj * 4 + d0 / 8, boff = (d0 % 8) * 2;
                const int lorow = e < kD ? p2::kLoRow + e : p2::kDenLo;   // hi row is e (kDenHi for e = D)
                *reinterpret_cast<uint32_t*>(dst + sw128_offset(e, chunk) + boff) = pack_bf16x2(h0, h1);
                *reinterpret_cast<uint32_t*>(dst + sw128_offset(lorow, chunk) + boff) =
                    pack_bf16x2(pv[k].x - h0, pv[k].y - h1);
            }
            fence_proxy_async_smem();
            mbar_arrive(&bfull[li & 1]);
            if (li + 1 < n) load_pre(li + 1);
        }
    } else if (warp >= 12) {
        // ------------------------------------------------ epilogues: warp w reads TMEM lane
        // quadrant q = w % 4 (query row n = 32 q + lane); its half hh = (w - 12) / 4 takes
        // key blocks {hh, hh + 2} of P (blocks after the quadrant are masked whole and
        // stay zero in P_s) and value columns 16 hh .. 16 hh + 15 of D.
        const int hh = (warp - 12) >> 2, q = warp & 3, nrow = 32 * q + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        const int64_t nsub = 2 * n;
        auto epi_a = [&](int64_t u) -> bool {
            const int tb = (int)(u % kTmemBufs), pb = (int)(u & 1);
            if (!mbar_wait(&pdone[tb], (uint32_t)(u / kTmemBufs) & 1, 916)) return false;
            if (u >= 2 && !mbar_wait(&u2done[pb], (uint32_t)((u >> 1) - 1) & 1, 917)) return false;
            tc_fence_after_sync();
            uint8_t* pbuf = ps + pb * kPsBuf;
            float rs = 0.f;
#pragma unroll 1
            for (int kk = 0; kk < 2; ++kk) {
                const int kc = hh + 2 * kk;                       // block of 32 keys
                if (kc > q) continue;
                float v[32];
                tmem_ld16(lane_base + tb * kBufCols + 32 * kc, v);
                tmem_ld16(lane_base + tb * kBufCols + 32 * kc + 16, v + 16);
                tmem_wait_ld();
                if (kc == q) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i > lane) v[i] = 0.f;
                }
                uint8_t* at = pbuf + (kc >> 1) * kPsAtom;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 w;
                    w.x = pack_bf16x2(v[8 * cc + 0], v[8 * cc + 1]);
                    w.y = pack_bf16x2(v[8 * cc + 2], v[8 * cc + 3]);
                    w.z = pack_bf16x2(v[8 * cc + 4], v[8 * cc + 5]);
                    w.w = pack_bf16x2(v[8 * cc + 6], v[8 * cc + 7]);
                    *reinterpret_cast<uint4*>(at + sw128_offset(nrow, (kc & 1) * 4 + cc)) = w;
                }
                float r4[4] = {0.f, 0.f, 0.f, 0.f};                // four chains
#pragma unroll
                for (int i = 0; i < 32; ++i) r4[i & 3] += v[i];
                rs += (r4[0] + r4[1]) + (r4[2] + r4[3]);
            }
            rowsum[((u % kTmemBufs) * 2 + hh) * kTok + nrow] = rs;
            tc_fence_before_sync();
            fence_proxy_async_smem();
            mbar_arrive(&psready[pb]);
            return true;
        };
        auto epi_b = [&](int64_t u) -> bool {
            const int64_t li = u >> 1;
            const int j = (int)(u & 1), tb = (int)(u % kTmemBufs);
            if (!mbar_wait(&mmadone[tb], (uint32_t)(u / kTmemBufs) & 1, 918)) return false;
            tc_fence_after_sync();
            const uint32_t ta = lane_base + tb * kBufCols;
            float hi[16], lo[16], den[2];
            tmem_ld16(ta + 16 * hh, hi);
            tmem_ld2(ta + p2::kDenHi, den);
            tmem_ld16(ta + p2::kLoRow + 16 * hh, lo);
            tmem_wait_ld();
            // the row sums of A(u) (this thread's and its partner warp's), read before the
            // buffer is handed back: A(u + 4) rewrites them once every thread has arrived
            if (!mbar_wait(&psready[u & 1], (uint32_t)(u >> 1) & 1, 919)) return false;
            const float intra = rowsum[(tb * 2 + 0) * kTok + nrow] + rowsum[(tb * 2 + 1) * kTok + nrow];
            tc_fence_before_sync();
            mbar_arrive(&tfree[tb]);
            const float inv = __frcp_rn(((den[0] + den[1]) + intra) + a.eps);
            uint8_t* ot = qring + (li % kQSlots) * kTile;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                float o[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) o[x] = (hi[8 * cc + x] + lo[8 * cc + x]) * inv;
                uint4 w;
                w.x = pack_bf16x2(o[0], o[1]);
                w.y = pack_bf16x2(o[2], o[3]);
                w.z = pack_bf16x2(o[4], o[5]);
                w.w = pack_bf16x2(o[6], o[7]);
                *reinterpret_cast<uint4*>(ot + sw128_offset(nrow, j * 4 + 2 * hh + cc)) = w;
            }
            fence_proxy_async_smem();
            mbar_arrive(&ofull[li % kQSlots]);
            return true;
        };
        for (int64_t u = 0; u < nsub && ok; ++u) {
            ok = epi_a(u);
            if (ok && u >= 1) ok = epi_b(u - 1);
        }
        if (ok && nsub > 0) ok = epi_b(nsub - 1);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace sana
