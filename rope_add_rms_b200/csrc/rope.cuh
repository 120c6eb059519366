// rope.cuh -- norm_rope kernels (RMS normalisation followed by the rotary embedding).
//
// Definitions: docs.rs nuvec-core 0.5.0, Enum FastOp, variants NormRope and Rope;
// docs.rs nuvec-nn 0.4.0 src/layers.rs, Rope (halves by default, base 10000, scale
// applied to positions).  Row k of x [B, H, L, D] sits at l = k mod L and is rotated
// at position offset + l: pair i turns by phi_i = (offset + l) * scale * theta_i with
// theta_i = base^(-2 i / dims); pairs are (i, i + dims/2) or, traditional, (2i, 2i + 1).
//
// Precision.  A pair output y_p = inv * (a_p cos - a_q sin), a = x * w, can cancel.
// A float32 angle (ulp(6000 rad) ~ 4.9e-4) or a float32 cos/sin (error 2^-24 |a|)
// misses the bfloat16 result by more than one ulp whenever |y_p| is much smaller
// than |a|.  So:
//   - each CTA builds the cos/sin of its positions in double precision (pow, sincos)
//     and keeps each as a float pair hi + lo (the split is exact to ~2^-48);
//   - a = x * w is exact in float32 for bfloat16 inputs (8 x 8 significant bits);
//   - the pair combination is evaluated with error-free products (fma), so the
//     float32 result is accurate to ~2^-23 relative plus ~2^-46 |a| absolute;
//   - the common factor inv = rsqrt(mean(x^2) + eps) multiplies last (a relative
//     error, harmless).
#pragma once

#include "async_copy.cuh"
#include "common.cuh"

namespace nvn {

struct RopeArgs {
    const void* x;
    const void* w;
    void* y;
    int64_t BH;         // rows / L
    int64_t L;
    int64_t offset;
    int64_t n_chunks;   // bh chunks per position
    int D;
    int nvec;           // 16-byte vectors per row
    int dims;
    int half;           // dims / 2
    int lpr;            // lanes per row (power of two <= 32), register path
    int bt;             // bh rows per CTA, register path
    float base;
    float scale;
    float eps;
    int normalize;
    int traditional;
    double log2_base;   // log2((double)base), computed on the host
    const float* freqs; // [dims/2] frequencies replacing base^(-2i/dims), or NULL
    int forward;        // 0: inverse rotation (-phi)
    int64_t y_len;      // rows per (b, h) in y: L, or the cache length
    int64_t y_off;      // first y row of a (b, h): 0, or offset in the cache form
};

// z = a_o * c + a_t * s for c = c_hi + c_lo, s = s_hi + s_lo (hi/lo float splits).
// t1 + e1 is a_t * s_hi exactly; the remaining products are ~2^-24 |a| and their own
// rounding is ~2^-48 |a|.
__device__ __forceinline__ float rotate_pair(float a_o, float a_t, float c_hi, float c_lo,
                                             float s_hi, float s_lo) {
    const float t1 = __fmul_rn(a_t, s_hi);
    const float e1 = __fmaf_rn(a_t, s_hi, -t1);
    const float z1 = __fmaf_rn(a_o, c_hi, t1);
    const float c2 = __fmaf_rn(a_t, s_lo, e1);
    const float c3 = __fmaf_rn(a_o, c_lo, c2);
    return __fadd_rn(z1, c3);
}

// cos and sin of phi_i = pos * scale * theta_i in double, split into float hi/lo, where
// theta_i = freqs[i] if a frequency vector is given, else base^(-2 i / dims) =
// 2^(-2 i log2(base) / dims).  The inverse rotation negates sin (exact).
__device__ __forceinline__ float4 angle_entry(const RopeArgs& a, double pos, int i) {
    const double theta = a.freqs ? (double)a.freqs[i]
                                 : exp2(-2.0 * (double)i / (double)a.dims * a.log2_base);
    const double phi = pos * (double)a.scale * theta;
    double s, c;
    sincos(phi, &s, &c);
    if (!a.forward) s = -s;
    const float ch = __double2float_rn(c);
    const float sh = __double2float_rn(s);
    return make_float4(ch, __double2float_rn(c - (double)ch), sh, __double2float_rn(s - (double)sh));
}

// The same on an element pair, in packed float32 arithmetic.
__device__ __forceinline__ float2 rotate_pair2(float2 a_o, float2 a_t, float2 c_hi, float2 c_lo,
                                               float2 s_hi, float2 s_lo) {
    const float2 t1 = mul2(a_t, s_hi);
    const float2 e1 = fma2(a_t, s_hi, neg2(t1));
    const float2 z1 = fma2(a_o, c_hi, t1);
    const float2 c2 = fma2(a_t, s_lo, e1);
    const float2 c3 = fma2(a_o, c_lo, c2);
    return add2(z1, c3);
}

// z = a_o * c - a_t * s on an element pair (the p side of halves pairing with the
// unsigned table), with the same error-free splitting.
__device__ __forceinline__ float2 rotate_sub2(float2 a_o, float2 a_t, float2 c_hi, float2 c_lo,
                                              float2 s_hi, float2 s_lo) {
    const float2 t1 = mul2(a_t, s_hi);
    const float2 e1 = fma2(a_t, s_hi, neg2(t1));  // a_t s_hi - t1, exact
    const float2 z1 = fma2(a_o, c_hi, neg2(t1));
    const float2 c2 = fma2(a_t, s_lo, e1);
    const float2 c3 = fma2(a_o, c_lo, neg2(c2));
    return add2(z1, c3);
}

// ---- register path ------------------------------------------------------------------
// One CTA = one position l and a chunk of bt rows (b, h) at that position, so the
// angle table of l is built once (dims/2 double sincos) and reused by all of them.
// A group of lpr lanes holds one row, one 16-byte vector per lane; each slot of the
// CTA takes rows slot, slot + slots, ...; kUnroll rows are loaded before any math.
// Halves pairing needs (dims/2) % VEC == 0: a lane's vector is then wholly the p side,
// wholly the q side or wholly past dims, and its partner vector sits hv = half/VEC
// lanes away (one shuffle per word).  Traditional pairs live inside one vector and need
// fewer registers: three CTAs per SM (measured 7% faster than two on bf16
// [8, 32, 2048, 128] with this kernel; the halves form loses at three, its spills cost
// more).  rope_pairs_kernel below serves both pairings where the rotated features fill an
// even number of whole vectors; this kernel takes the other shapes with dims < D and plans
// that ask for one vector per lane.
template <typename T, bool TRAD>
__global__ void __launch_bounds__(256, TRAD ? 3 : 2) rope_rows_kernel(const RopeArgs a) {
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    constexpr int kUnroll = 4;
    extern __shared__ float4 tab[];  // [half]: (cos_hi, cos_lo, sin_hi, sin_lo)

    const int64_t chunk = blockIdx.x % a.n_chunks;
    const int64_t l = blockIdx.x / a.n_chunks;
    const int lpr = a.lpr;
    const int lane = threadIdx.x & (lpr - 1);  // vector index within the row
    const int slot = threadIdx.x / lpr;
    const int slots = blockDim.x / lpr;
    const int v = lane;
    const bool has_vec = v < a.nvec;
    const int hv = a.half / VEC;  // halves: partner distance in vectors

    // partner vector (halves) and the sign of sin for this lane's elements
    int pv = v;
    if (!TRAD) pv = (v < hv) ? v + hv : (v < 2 * hv ? v - hv : v);

    const bool norm = a.normalize != 0;

    // first rows' loads go out before the table is built
    const int64_t bh0 = chunk * (int64_t)a.bt;
    const int64_t bh_end = min(bh0 + (int64_t)a.bt, a.BH);
    const size_t row_bytes = (size_t)a.D * sizeof(T);
    const size_t lstride = (size_t)a.L * row_bytes;  // between consecutive bh at fixed l
    const char* xbase = static_cast<const char*>(a.x) + (size_t)l * row_bytes + (size_t)v * 16;
    // y row of (b, h, l): b * y_len + y_off + l (y_len = L, y_off = 0 unless a cache)
    const size_t ystride = (size_t)a.y_len * row_bytes;
    char* ybase = static_cast<char*>(a.y) + (size_t)(a.y_off + l) * row_bytes + (size_t)v * 16;

    pdl_wait();
    pdl_release();
    // Every thread runs the same trip count (rows past bh_end are predicated off):
    // the shuffles below involve the whole warp, which may hold several rows.
    // The first rows' loads go out before the angle table is built, so its latency
    // (double exp2 and sincos) hides behind theirs.
    V16 xv[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t b = bh0 + slot + (int64_t)u * slots;
        if (has_vec && b < bh_end) xv[u] = ld_stream(xbase + (size_t)b * lstride);
    }
    // per-column weights of this lane's elements and of their partners
    const V16 w_own_v = (norm && a.w && has_vec)
                            ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16)
                            : ones_vec<T>();
    V16 w_par_v = w_own_v;
    if (!TRAD && pv != v && norm && a.w && pv < a.nvec)
        w_par_v = ld_param(static_cast<const char*>(a.w) + (size_t)pv * 16);
    const double pos = (double)(a.offset + l);
    for (int i = threadIdx.x; i < a.half; i += blockDim.x)
        tab[i] = angle_entry(a, pos, i);
    float2 w_own[VEC / 2], w_par[VEC / 2];
#pragma unroll
    for (int e = 0; e < VEC; e += 2) {
        w_own[e / 2] = E::get2(w_own_v, e);
        w_par[e / 2] = E::get2(w_par_v, e);
    }
    __syncthreads();

    // this lane's table entries, sin already carrying the sign of its side; elements
    // past dims get the identity (cos 1, sin 0) and the scalar path below
    float2 c_hi[VEC / 2], c_lo[VEC / 2], s_hi[VEC / 2], s_lo[VEC / 2];
    bool all_rot = has_vec;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        const int j = v * VEC + e;
        const bool r = has_vec && j < a.dims;
        all_rot = all_rot && r;
        int i = 0;
        float sg = 1.f;
        if (TRAD) {
            i = j >> 1;
            sg = (j & 1) ? 1.f : -1.f;
        } else {
            i = (j < a.half) ? j : j - a.half;
            sg = (j < a.half) ? -1.f : 1.f;
        }
        float4 t4 = make_float4(1.f, 0.f, 0.f, 0.f);
        if (r) t4 = tab[i];
        float* ch = reinterpret_cast<float*>(&c_hi[e / 2]);
        float* cl = reinterpret_cast<float*>(&c_lo[e / 2]);
        float* sh = reinterpret_cast<float*>(&s_hi[e / 2]);
        float* sl = reinterpret_cast<float*>(&s_lo[e / 2]);
        ch[e & 1] = t4.x;
        cl[e & 1] = t4.y;
        sh[e & 1] = sg * t4.z;
        sl[e & 1] = sg * t4.w;
    }

    const float invD = 1.0f / (float)a.D;
    for (int64_t base = bh0; base < bh_end; base += (int64_t)kUnroll * slots) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t b = base + slot + (int64_t)u * slots;
            const bool live = has_vec && b < bh_end;
            V16 xo = live ? xv[u] : zeros_vec<T>();
            // the next round's load for this unroll slot goes out now
            const int64_t bn = b + (int64_t)kUnroll * slots;
            if (has_vec && bn < bh_end) xv[u] = ld_stream(xbase + (size_t)bn * lstride);

            float2 x2[VEC / 2];
            float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < VEC; e += 2) {
                x2[e / 2] = E::get2(xo, e);
                ss2 = fma2(x2[e / 2], x2[e / 2], ss2);
            }
            const float ss = group_sum(__fadd_rn(ss2.x, ss2.y), lpr);
            const float inv = norm ? rsqrtf(__fmaf_rn(ss, invD, a.eps)) : 1.f;
            const float2 inv2 = make_float2(inv, inv);

            V16 xp = xo;  // partner words
            if (!TRAD) {
                const int src = pv & (lpr - 1);
#pragma unroll
                for (int q = 0; q < 4; ++q) xp.u[q] = __shfl_sync(0xFFFFFFFFu, xo.u[q], src, lpr);
            }
            if (live) {
                // a = x * w, exact in float32 for bfloat16 data; each product formed once
                float2 ao[VEC / 2], at[VEC / 2];
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    ao[e / 2] = mul2(x2[e / 2], w_own[e / 2]);
                    if (TRAD)
                        at[e / 2] = make_float2(ao[e / 2].y, ao[e / 2].x);
                    else
                        at[e / 2] = mul2(E::get2(xp, e), w_par[e / 2]);
                }
                V16 o;
                if (all_rot) {
#pragma unroll
                    for (int e = 0; e < VEC; e += 2) {
                        const int q = e / 2;
                        const float2 z =
                            rotate_pair2(ao[q], at[q], c_hi[q], c_lo[q], s_hi[q], s_lo[q]);
                        E::put2(o, e, mul2(z, inv2));
                    }
                } else {
                    // a vector holding features past dims: those keep a = x * w
#pragma unroll
                    for (int e = 0; e < VEC; ++e) {
                        const int q = e / 2;
                        const float* aof = reinterpret_cast<const float*>(&ao[q]);
                        const float* atf = reinterpret_cast<const float*>(&at[q]);
                        const float* ch = reinterpret_cast<const float*>(&c_hi[q]);
                        const float* cl = reinterpret_cast<const float*>(&c_lo[q]);
                        const float* sh = reinterpret_cast<const float*>(&s_hi[q]);
                        const float* sl = reinterpret_cast<const float*>(&s_lo[q]);
                        const int h = e & 1;
                        const int j = v * VEC + e;
                        float z = aof[h];
                        if (j < a.dims) z = rotate_pair(aof[h], atf[h], ch[h], cl[h], sh[h], sl[h]);
                        const float y = __fmul_rn(z, inv);
                        if (h)
                            E::put2(o, e - 1, E::get(o, e - 1), y);
                        else
                            E::put2(o, e, y, 0.f);
                    }
                }
                st_stream(ybase + (size_t)b * ystride, o);
            }
        }
    }
}

// ---- register path, two vectors per lane ---------------------------------------------------
// Each lane holds vectors v and v + nvec/2 of a row (16-byte vectors, nvec even) and keeps
// its elements as float pairs of rotation partners: p[k] holds the first members (the
// cos-side inputs of y_p = a_p cos - a_q sin) of two pairs and q[k] their second members,
// so one packed rotation serves two pairs and no partner is in another lane.  With dims < D
// (pair_lane_vectors) the rotated lanes pair vectors v and v + dims/(2 VEC) instead and the
// other lanes hold the features past dims.
//   halves:      vector v holds the p members of pairs v*VEC .. v*VEC + VEC - 1 and
//                vector v + nvec/2 their q members;
//   traditional: each vector holds VEC/2 whole pairs (2i, 2i + 1).
// The angle table and the lane's weights stay in shared memory as records of two pairs,
// transposed so that the lanes of a row read consecutive records, and are read per row:
// with neither in registers four CTAs fit per SM (three for float32), and a record load
// yields the float pairs the packed rotation takes.  Halves, bf16 [8, 32, 2048, 128], with
// the lanes per row taken from the arguments: 51.7 us; 54.3 us with the weights in registers
// (3 CTAs/SM), 59.2 us with one table entry per pair, 69.5 us with the table in registers
// (2 CTAs/SM).  With the lanes per row fixed at compile time (rope_pairs_kernel's HV):
// 48.1-48.3 us.
template <typename T, bool TRAD>
struct PairLayout {
    using E = Elem<T>;
    static constexpr int VEC = E::kVec;
    static constexpr int NP = VEC / 2;  // float pairs per side
    // vector (0: v, 1: v + nvec/2) and element of the .x (h = 0) or .y (h = 1) member of
    // slot k on side s (0: p, 1: q)
    __device__ __forceinline__ static void where(int k, int h, int s, int& vec, int& e) {
        if (!TRAD) {
            vec = s;
            e = 2 * k + h;
        } else {
            vec = k < NP / 2 ? 0 : 1;
            e = 2 * (2 * (k % (NP / 2)) + h) + s;
        }
    }
    // The table holds one record per two pairs served by one packed rotation: C =
    // (cos_hi, cos_hi', cos_lo, cos_lo') and S = (sin_hi, sin_hi', sin_lo, sin_lo'), so one
    // 16-byte load gives the float pairs directly.  Records are transposed (row k of
    // `lanes` records), so the lanes of a row read consecutive records:
    //   halves:      slot k of lane v  -> record k * nvec/2 + v;
    //   traditional: slot k of lane v  -> record (k mod NP/2) * nvec + (v or v + nvec/2).
    __device__ __forceinline__ static int record(int v0, int v1, int k, int hvec) {
        if (!TRAD) return k * hvec + v0;
        return (k % (NP / 2)) * (2 * hvec) + (k < NP / 2 ? v0 : v1);
    }
    // record of rotation pair i and which member (.x / .y of each half) it is
    __device__ __forceinline__ static int record_of(int i, int hvec, int& h) {
        if (!TRAD) {
            h = (i % VEC) & 1;
            return ((i % VEC) >> 1) * hvec + i / VEC;
        }
        h = (i % NP) & 1;
        return ((i % NP) >> 1) * (2 * hvec) + i / NP;
    }
    __device__ __forceinline__ static void split(const V16& a, const V16& b, float2 (&p)[NP],
                                                 float2 (&q)[NP]) {
#pragma unroll
        for (int k = 0; k < NP; ++k)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                int vp, ep, vq, eq;
                where(k, h, 0, vp, ep);
                where(k, h, 1, vq, eq);
                reinterpret_cast<float*>(&p[k])[h] = E::get(vp ? b : a, ep);
                reinterpret_cast<float*>(&q[k])[h] = E::get(vq ? b : a, eq);
            }
    }
    __device__ __forceinline__ static void join(const float2 (&p)[NP], const float2 (&q)[NP],
                                                V16& a, V16& b) {
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            if (!TRAD) {
                E::put2(a, 2 * k, p[k]);
                E::put2(b, 2 * k, q[k]);
            } else {  // pair (2i, 2i + 1) is elements (e, e + 1) of one vector
                V16& v = k < NP / 2 ? a : b;
                const int e0 = 4 * (k % (NP / 2));
                E::put2(v, e0, p[k].x, q[k].x);
                E::put2(v, e0 + 2, p[k].y, q[k].y);
            }
        }
    }
};

// The angle records of position offset + l, written by threads t = 0, n, 2n, ... < half:
// C [half / 2] then S [half / 2], each record serving two pairs (PairLayout::record_of).
template <typename T, bool TRAD>
__device__ __forceinline__ void build_angle_records(const RopeArgs& a, float4* ctab, int64_t l,
                                                    int t, int n) {
    using PL = PairLayout<T, TRAD>;
    const double pos = (double)(a.offset + l);
    float* tabf = reinterpret_cast<float*>(ctab);
    const int nrec = a.half / 2;
    const int hr = a.half / PL::VEC;  // lanes of a row that rotate (all of them when dims == D)
    for (int i = t; i < a.half; i += n) {
        int h = 0;
        const int rec = PL::record_of(i, hr, h);
        const float4 e = angle_entry(a, pos, i);
        tabf[rec * 4 + h] = e.x;               // C: cos_hi, cos_lo
        tabf[rec * 4 + 2 + h] = e.y;
        tabf[(nrec + rec) * 4 + h] = e.z;      // S: sin_hi, sin_lo
        tabf[(nrec + rec) * 4 + 2 + h] = e.w;
    }
}

// The lanes' weight records W [NP][lanes], record k * lanes + lane; lanes with a vector
// (has_vec) read w at their vectors v0 and v1, and those of slot 0 (write) store the records.
template <typename T, bool TRAD>
__device__ __forceinline__ void store_weight_records(const RopeArgs& a, float4* wtab, int lane,
                                                     int lanes, int v0, int v1, bool has_vec,
                                                     bool write) {
    using PL = PairLayout<T, TRAD>;
    constexpr int NP = PL::NP;
    const bool has_w = a.normalize != 0 && a.w != nullptr && has_vec;
    const V16 wa = has_w ? ld_param(static_cast<const char*>(a.w) + (size_t)v0 * 16) : ones_vec<T>();
    const V16 wb = has_w ? ld_param(static_cast<const char*>(a.w) + (size_t)v1 * 16) : ones_vec<T>();
    float2 wp[NP], wq[NP];
    PL::split(wa, wb, wp, wq);
    if (write)
#pragma unroll
        for (int k = 0; k < NP; ++k)
            wtab[k * lanes + lane] = make_float4(wp[k].x, wp[k].y, wq[k].x, wq[k].y);
}

// One row of the two-vectors-per-lane layout: sum of squares over the lane group, then the
// rotation of this lane's pairs, weights applied first and the row's 1/rms last.  Every
// lane of the group takes part (the group sum); lanes with live == false store nothing.
// hvec = nvec / 2 vectors a lane group covers per side (the weight records' stride: record
// k * hvec + lane), lpr lanes per row; hr of the lanes rotate (hr = hvec when dims == D) and
// the table holds hr * NP C records, then as many S records; a lane with rot == false holds
// two vectors past dims, which keep a = x w and take the row's 1/rms.  PART selects how:
//   0  dims == D, every lane rotates;
//   1  the lanes past dims branch off to a scaling loop (cheaper while fewer than half the
//      lanes of a row rotate: the rotating loop then runs on few lanes);
//   2  every lane runs the rotating loop, those past dims on lane 0's records (a broadcast)
//      and keeping their weighted inputs by a select, so the result is exactly a = x w
//      whatever the discarded rotation gives; one instruction stream, each weight record
//      read once.
// Measured, bf16 [8, 32, 2048, 128], ring of 3 rounds: dims 32 / 64 / 96 with form 1
// 45.9 / 51.6 / 48.7 us, with form 2 47.6 / 47.7 / 47.8 us.
template <typename T, bool TRAD, int PART>
__device__ __forceinline__ void rope_pairs_row(const RopeArgs& a, const float4* ctab,
                                               const float4* wtab, const V16& xa, const V16& xb,
                                               bool live, int lane, int v0, int v1, int hvec,
                                               int hr, bool rot, int lpr, float invD,
                                               char* yrow) {
    using PL = PairLayout<T, TRAD>;
    constexpr int NP = PL::NP;
    float2 p[NP], q[NP];
    PL::split(xa, xb, p, q);
    float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        ss2 = fma2(p[k], p[k], ss2);
        ss2 = fma2(q[k], q[k], ss2);
    }
    const float ss = group_sum(__fadd_rn(ss2.x, ss2.y), lpr);
    const float inv = a.normalize ? rsqrtf(__fmaf_rn(ss, invD, a.eps)) : 1.f;
    const float2 inv2 = make_float2(inv, inv);
    if (live) {  // only lanes holding vectors read the table
        float2 yp[NP], yq[NP];
        if (PART == 2) {
            // every lane rotates: a lane past dims reads lane 0's records of the slot (a
            // broadcast) and keeps its weighted inputs by a select
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                const int rec = PL::record(rot ? v0 : 0, rot ? v1 : hr, k, hr);
                const float4 c4 = ctab[rec], s4 = ctab[hr * NP + rec];
                const float2 ch = make_float2(c4.x, c4.y), cl = make_float2(c4.z, c4.w);
                const float2 sh = make_float2(s4.x, s4.y), sl = make_float2(s4.z, s4.w);
                const float4 w4 = wtab[k * hvec + lane];
                const float2 ap = mul2(p[k], make_float2(w4.x, w4.y));
                const float2 aq = mul2(q[k], make_float2(w4.z, w4.w));
                const float2 rp = rotate_sub2(ap, aq, ch, cl, sh, sl);
                const float2 rq = rotate_pair2(aq, ap, ch, cl, sh, sl);
                yp[k] = mul2(rot ? rp : ap, inv2);
                yq[k] = mul2(rot ? rq : aq, inv2);
            }
        } else if (rot) {
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                const int rec = PL::record(v0, v1, k, hr);
                const float4 c4 = ctab[rec], s4 = ctab[hr * NP + rec];
                const float2 ch = make_float2(c4.x, c4.y), cl = make_float2(c4.z, c4.w);
                const float2 sh = make_float2(s4.x, s4.y), sl = make_float2(s4.z, s4.w);
                const float4 w4 = wtab[k * hvec + lane];
                const float2 ap = mul2(p[k], make_float2(w4.x, w4.y));  // exact for bf16 data
                const float2 aq = mul2(q[k], make_float2(w4.z, w4.w));
                yp[k] = mul2(rotate_sub2(ap, aq, ch, cl, sh, sl), inv2);
                yq[k] = mul2(rotate_pair2(aq, ap, ch, cl, sh, sl), inv2);
            }
        } else {  // past dims, lanes diverged from the rotating ones: a = x w, then 1/rms
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                const float4 w4 = wtab[k * hvec + lane];
                yp[k] = mul2(mul2(p[k], make_float2(w4.x, w4.y)), inv2);
                yq[k] = mul2(mul2(q[k], make_float2(w4.z, w4.w)), inv2);
            }
        }
        V16 o0, o1;
        PL::join(yp, yq, o0, o1);
        st_stream(yrow + (size_t)v0 * 16, o0);
        st_stream(yrow + (size_t)v1 * 16, o1);
    }
}

// rows in flight per lane group (measured best of 2..4 at three or four CTAs per SM: 2 for
// bfloat16, 4 for the float32 rows that carry twice the bytes per element)
template <typename T>
__host__ __device__ constexpr int rope_pairs_unroll() { return sizeof(T) == 4 ? 4 : 2; }

// One CTA of kRopeThreads per (position l, chunk of bt rows): the table of l is built while
// the chunk's first rows load.  HV > 0 fixes hvec = nvec / 2 = lanes per row at compile time
// (4, 8 or 16: D = 128 in bfloat16 is 8), so every table and row offset is a constant and
// the group sum a fixed butterfly; HV = 0 takes them from the arguments.
constexpr int kRopeThreads = 256;

// PART (dims < D, HV > 0 only): the first hr = dims / (2 VEC) lanes of a row hold the
// rotated vectors as partner pairs (lane j: vectors j and j + hr), the others two of the
// vectors past dims each (lane j: R + j - hr and that plus (nvec - R) / 2, R = dims / VEC).
template <bool PART, int HV>
__device__ __forceinline__ void pair_lane_vectors(const RopeArgs& a, int lane, int hvec, int vec,
                                                  int& hr, int& v0, int& v1, bool& rot) {
    if (!PART) {
        hr = hvec;
        v0 = lane;
        v1 = lane + hvec;
        rot = true;
        return;
    }
    hr = a.half / vec;
    rot = lane < hr;
    const int R = 2 * hr;
    v0 = rot ? lane : R + lane - hr;
    v1 = rot ? lane + hr : v0 + (a.nvec - R) / 2;
}

template <typename T, bool TRAD, int HV, int PART = 0>
__global__ void __launch_bounds__(kRopeThreads, sizeof(T) == 2 ? 4 : 3)
    rope_pairs_kernel(const RopeArgs a) {
    constexpr int kUnroll = rope_pairs_unroll<T>();
    constexpr int NP = PairLayout<T, TRAD>::NP;
    // records: C [hvec NP], S [hvec NP], then the lanes' weights W [NP][hvec]
    extern __shared__ float4 tab[];

    const int64_t chunk = blockIdx.x % a.n_chunks;
    const int64_t l = blockIdx.x / a.n_chunks;
    const int hvec = HV > 0 ? HV : a.nvec / 2;
    const int lpr = HV > 0 ? HV : a.lpr;
    const int lane = threadIdx.x & (lpr - 1);
    const int slot = threadIdx.x / lpr;
    const int slots = kRopeThreads / lpr;
    static_assert(PART == 0 || HV > 0, "dims < D takes the fixed-lane kernels");
    int hr, v0, v1;
    bool rot;
    pair_lane_vectors<PART != 0, HV>(a, lane, hvec, Elem<T>::kVec, hr, v0, v1, rot);
    // with HV fixed every lane of a group holds vectors (lpr == hvec)
    const bool has_vec = HV > 0 || lane < hvec;

    pdl_wait();
    pdl_release();

    const int64_t bh0 = chunk * (int64_t)a.bt;
    const int64_t bh_end = min(bh0 + (int64_t)a.bt, a.BH);
    const size_t row_bytes = (size_t)a.D * sizeof(T);
    const size_t lstride = (size_t)a.L * row_bytes;
    const char* xbase = static_cast<const char*>(a.x) + (size_t)l * row_bytes;
    const size_t ystride = (size_t)a.y_len * row_bytes;
    char* ybase = static_cast<char*>(a.y) + (size_t)(a.y_off + l) * row_bytes;

    V16 xv[kUnroll][2];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t b = bh0 + slot + (int64_t)u * slots;
        xv[u][0] = zeros_vec<T>();
        xv[u][1] = zeros_vec<T>();
        if (has_vec && b < bh_end) {
            xv[u][0] = ld_stream(xbase + (size_t)b * lstride + (size_t)v0 * 16);
            xv[u][1] = ld_stream(xbase + (size_t)b * lstride + (size_t)v1 * 16);
        }
    }
    // the angle table (half records) is built while the first rows' loads are in flight
    float4* wtab = tab + 2 * hr * NP;
    build_angle_records<T, TRAD>(a, tab, l, threadIdx.x, kRopeThreads);
    store_weight_records<T, TRAD>(a, wtab, lane, hvec, v0, v1, has_vec, slot == 0 && has_vec);
    __syncthreads();

    const float invD = 1.0f / (float)a.D;
    for (int64_t base = bh0; base < bh_end; base += (int64_t)kUnroll * slots) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t b = base + slot + (int64_t)u * slots;
            const bool live = has_vec && b < bh_end;
            // a row past the chunk is reduced from stale registers and not stored; lanes
            // without a vector keep the zeros they started with, so add nothing to the sum
            const V16 xa = xv[u][0];
            const V16 xb = xv[u][1];
            const int64_t bn = b + (int64_t)kUnroll * slots;
            if (has_vec && bn < bh_end) {
                xv[u][0] = ld_stream(xbase + (size_t)bn * lstride + (size_t)v0 * 16);
                xv[u][1] = ld_stream(xbase + (size_t)bn * lstride + (size_t)v1 * 16);
            }
            rope_pairs_row<T, TRAD, PART>(a, tab, wtab, xa, xb, live, lane, v0, v1, hvec, hr, rot,
                                          lpr, invD, ybase + (size_t)b * ystride);
        }
    }
}

// The same rows with DEPTH rounds of loads in flight per lane group, staged by per-thread
// asynchronous copies (cp.async, 16 bytes, L2 only) into a ring of shared memory instead of
// registers, so rows in flight cost shared memory (DEPTH x 8 KB a CTA) rather than the
// registers that hold four CTAs per SM.  Each thread copies, waits for and reads back only
// its own two vectors of a round (slot [round % DEPTH][vector][thread]: consecutive
// threads, consecutive 16 bytes), so no barrier is needed: cp.async.wait_group orders a
// thread's own copies, one commit group per round (empty past the chunk's last row).  A
// slot is refilled only after the row read from it has been computed.
// shared memory of rope_pairs_async_kernel: the table and weight records, then the ring
__host__ __device__ constexpr size_t rope_async_ring_bytes(int depth) {
    return (size_t)depth * 2 * kRopeThreads * 16;
}

template <typename T, bool TRAD, int HV, int DEPTH, int PART = 0>
__global__ void __launch_bounds__(kRopeThreads, sizeof(T) == 2 ? 4 : 3)
    rope_pairs_async_kernel(const RopeArgs a) {
    static_assert(HV > 0, "lanes per row fixed at compile time");
    constexpr int NP = PairLayout<T, TRAD>::NP;
    constexpr int kSlots = kRopeThreads / HV;
    const int lane = threadIdx.x & (HV - 1);
    const int slot = threadIdx.x / HV;
    int hr, v0, v1;
    bool rot;
    pair_lane_vectors<PART != 0, HV>(a, lane, HV, Elem<T>::kVec, hr, v0, v1, rot);
    // records: C [hr NP], S [hr NP], the lanes' weights W [NP][HV], then the ring
    extern __shared__ float4 tab[];
    float4* wtab = tab + 2 * hr * NP;
    V16* ring = reinterpret_cast<V16*>(wtab + NP * HV);

    const int64_t chunk = blockIdx.x % a.n_chunks;
    const int64_t l = blockIdx.x / a.n_chunks;

    pdl_wait();
    pdl_release();

    const int64_t bh0 = chunk * (int64_t)a.bt;
    const int64_t bh_end = min(bh0 + (int64_t)a.bt, a.BH);
    const size_t row_bytes = (size_t)a.D * sizeof(T);
    const size_t lstride = (size_t)a.L * row_bytes;
    const char* xbase = static_cast<const char*>(a.x) + (size_t)l * row_bytes;
    const size_t ystride = (size_t)a.y_len * row_bytes;
    char* ybase = static_cast<char*>(a.y) + (size_t)(a.y_off + l) * row_bytes;
    const int rounds = (a.bt + kSlots - 1) / kSlots;

    auto issue = [&](int r) {
        const int64_t b = bh0 + slot + (int64_t)r * kSlots;
        if (r < rounds && b < bh_end) {
            const char* src = xbase + (size_t)b * lstride;
            V16* dst = ring + (size_t)(r % DEPTH) * 2 * kRopeThreads + threadIdx.x;
            cp_async16(dst, src + (size_t)v0 * 16);
            cp_async16(dst + kRopeThreads, src + (size_t)v1 * 16);
        }
        cp_async_commit();
    };
#pragma unroll
    for (int r = 0; r < DEPTH; ++r) issue(r);
    // the angle table is built while the first rounds load
    build_angle_records<T, TRAD>(a, tab, l, threadIdx.x, kRopeThreads);
    store_weight_records<T, TRAD>(a, wtab, lane, HV, v0, v1, true, slot == 0);
    __syncthreads();

    const float invD = 1.0f / (float)a.D;
    for (int r = 0; r < rounds; ++r) {
        cp_async_wait<DEPTH - 1>();  // this thread's copies of round r have landed
        const V16* src = ring + (size_t)(r % DEPTH) * 2 * kRopeThreads + threadIdx.x;
        const V16 xa = src[0];
        const V16 xb = src[kRopeThreads];
        const int64_t b = bh0 + slot + (int64_t)r * kSlots;
        // a row past the chunk is reduced from stale shared memory and not stored
        rope_pairs_row<T, TRAD, PART>(a, tab, wtab, xa, xb, b < bh_end, lane, v0, v1, HV, hr,
                                      rot, HV, invD, ybase + (size_t)b * ystride);
        issue(r + DEPTH);
    }
    cp_async_wait<0>();
}

// ---- generic path ---------------------------------------------------------------------
// Any D, dims and alignment: one CTA per row.  Pass 1: sum of squares.  Pass 2: each
// thread takes whole pairs (reads both members, then writes both, so y may be x) with
// its angle computed in double, then the features past dims.
template <typename T>
__global__ void __launch_bounds__(128) rope_generic_kernel(const RopeArgs a) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    __shared__ float red[2][32];
    const int nw = blockDim.x >> 5;
    const bool norm = a.normalize != 0;
    const int64_t rows = a.BH * a.L;
    int it = 0;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x, ++it) {
        const int64_t r0 = row * (int64_t)a.D;
        float inv = 1.f;
        if (norm) {
            float ss = 0.f;
            for (int j = threadIdx.x; j < a.D; j += blockDim.x) {
                const float f = E::load1(a.x, r0 + j);
                ss = fmaf(f, f, ss);
            }
            ss = warp_sum(ss);
            float* buf = red[it & 1];
            if ((threadIdx.x & 31) == 0) buf[threadIdx.x >> 5] = ss;
            __syncthreads();
            ss = 0.f;
            for (int i = 0; i < nw; ++i) ss += buf[i];
            inv = rsqrtf(__fmaf_rn(ss, 1.0f / (float)a.D, a.eps));
        }
        const double pos = (double)(a.offset + row % a.L);
        const int64_t o0 = ((row / a.L) * a.y_len + a.y_off + row % a.L) * (int64_t)a.D;
        for (int i = threadIdx.x; i < a.half; i += blockDim.x) {
            const int p = a.traditional ? 2 * i : i;
            const int q = a.traditional ? 2 * i + 1 : i + a.half;
            const float wp = (norm && a.w) ? E::load1(a.w, p) : 1.f;
            const float wq = (norm && a.w) ? E::load1(a.w, q) : 1.f;
            const float ap = __fmul_rn(E::load1(a.x, r0 + p), wp);
            const float aq = __fmul_rn(E::load1(a.x, r0 + q), wq);
            const float4 t = angle_entry(a, pos, i);
            const float yp = rotate_pair(ap, aq, t.x, t.y, -t.z, -t.w);
            const float yq = rotate_pair(aq, ap, t.x, t.y, t.z, t.w);
            E::store1(a.y, o0 + p, __fmul_rn(yp, inv));
            E::store1(a.y, o0 + q, __fmul_rn(yq, inv));
        }
        for (int j = a.dims + threadIdx.x; j < a.D; j += blockDim.x) {
            const float wj = (norm && a.w) ? E::load1(a.w, j) : 1.f;
            E::store1(a.y, o0 + j, __fmul_rn(__fmul_rn(E::load1(a.x, r0 + j), wj), inv));
        }
    }
}

}  // namespace nvn
