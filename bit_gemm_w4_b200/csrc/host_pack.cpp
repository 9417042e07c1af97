// Host-side disaggregation W ~= Q(W) + R and the packed device layout.
//
// MosaicQuant (gist.science/paper/2606.15652), "Methodology" 1.: the weight
// matrix is split into a dense 4-bit base that captures the inliers and a
// sparse 4-bit residual that compensates the quantization error of the
// outliers. The encoding (int4 asymmetric, group 128, fp16 scale and zero per
// group; per-row top-k |error| residual as int4 CSR with one fp16 scale per
// row) is fixed by this library; every step is done in fp64 with
// round-half-to-even so the result is reproducible bit for bit:
//   lo = min(min v, 0), hi = max(max v, 0), s = fp16((hi - lo) / 15)
//   (1 for an all-zero group, 2^-24 if it rounds to 0), z = clamp(rne(-lo/s)),
//   q = clamp(rne(v/s) + z, 0, 15); E = v - (q - z) s; the k_n largest |E| of
//   a row (ties to the smaller column) become the residual with
//   s_r = fp16(max|E| / 7) (1 if 0) and q_r = clamp(rne(E/s_r), -8, 7).
// No CUDA call is made in this file.

#include <algorithm>
#include <cfenv>
#include <cmath>
#include <cstring>
#include <numeric>
#include <thread>

#include "internal.h"

namespace mq {

uint16_t f64_to_f16_bits(double x) {
    uint16_t sign = std::signbit(x) ? 0x8000 : 0;
    double a = std::fabs(x);
    if (std::isnan(x)) return sign | 0x7E00;
    // 65520 is halfway between the largest finite fp16 (65504) and 2^16;
    // the tie goes to the even pattern, which is the overflow to inf.
    if (a >= 65520.0) return sign | 0x7C00;
    if (a < std::ldexp(1.0, -14)) {
        // subnormal range: value = m * 2^-24, m in [0, 1024]; m = 1024 is
        // the smallest normal and has the same bit pattern.
        double m = std::nearbyint(std::ldexp(a, 24));
        return sign | static_cast<uint16_t>(m);
    }
    int e;
    std::frexp(a, &e);  // a = f * 2^e, f in [0.5, 1)
    e -= 1;             // a = (2f) * 2^e, 2f in [1, 2)
    double m = std::nearbyint(std::ldexp(a, 10 - e));  // in [1024, 2048]
    if (m == 2048.0) {
        m = 1024.0;
        e += 1;
    }
    return sign | static_cast<uint16_t>(((e + 15) << 10) | (static_cast<int>(m) - 1024));
}

double f16_bits_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1, ex = (h >> 10) & 0x1F, man = h & 0x3FF;
    double v;
    if (ex == 0)
        v = std::ldexp(static_cast<double>(man), -24);
    else if (ex == 31)
        v = man ? NAN : INFINITY;
    else
        v = std::ldexp(static_cast<double>(man + 1024), ex - 25);
    return sign ? -v : v;
}

int64_t residual_count(int64_t K, double rho) {
    return static_cast<int64_t>(std::floor(rho * static_cast<double>(K) + 0.5));
}

mq_status check_shape(int64_t N, int64_t K, const mq_pack_opts *opts) {
    if (!opts) return fail(MQ_ERR_INVALID_ARG, "opts is NULL");
    if (opts->group_size != kGroup)
        return fail(MQ_ERR_UNSUPPORTED, "only group_size 128 is supported");
    if (N <= 0 || K <= 0) return fail(MQ_ERR_INVALID_ARG, "N and K must be positive");
    if (K % kGroup) return fail(MQ_ERR_INVALID_ARG, "K must be a multiple of 128");
    if (K > 65536) return fail(MQ_ERR_INVALID_ARG, "K must be at most 65536 (u16 columns)");
    if (N > (int64_t(1) << 31) - 1) return fail(MQ_ERR_INVALID_ARG, "N too large");
    if (opts->residual_blocks == 0) {
        double rho = opts->residual_density;
        if (!(rho >= 0.0 && rho <= 1.0))
            return fail(MQ_ERR_INVALID_ARG, "residual_density must be in [0, 1]");
    } else if (opts->residual_blocks == 1) {
        double f = opts->block_fraction;
        if (!(f >= 0.0 && f <= 1.0)) return fail(MQ_ERR_INVALID_ARG, "block_fraction must be in [0, 1]");
        if (N % kBlockRows) return fail(MQ_ERR_INVALID_ARG, "block mode needs N % 16 == 0");
        if (opts->channel_weight)
            for (int64_t k = 0; k < K; ++k) {
                const double h = opts->channel_weight[k];
                if (!(std::isfinite(h) && h >= 0.0))
                    return fail(MQ_ERR_INVALID_ARG, "channel weights must be finite and >= 0");
            }
    } else {
        return fail(MQ_ERR_UNSUPPORTED, "unknown residual_blocks mode");
    }
    return MQ_OK;
}

int64_t residual_blocks_selected(int64_t N, int64_t K, double fraction) {
    const int64_t blocks = (N / kBlockRows) * (K / kBlockCols);
    return static_cast<int64_t>(std::floor(fraction * static_cast<double>(blocks) + 0.5));
}

namespace {

struct RowError {
    bool bad = false;
    std::string msg;
};

// D1 and D2 for row n: codes, scales and zero points into d, the errors
// E = w - deq into E[0..K). Returns false (with err set) on bad input.
bool base_row(const float *W, int64_t K, int64_t n, HostDecomp &d, double *E, RowError &err) {
    const int64_t G = K / kGroup;
    {
        const float *w = W + n * K;
        uint8_t *q = d.q.data() + n * K;
        for (int64_t g = 0; g < G; ++g) {
            const float *v = w + g * kGroup;
            double lo = 0.0, hi = 0.0;
            for (int j = 0; j < kGroup; ++j) {
                double x = static_cast<double>(v[j]);
                if (!std::isfinite(x)) {
                    err.bad = true;
                    err.msg = "W holds NaN or Inf";
                    return false;
                }
                lo = std::min(lo, x);
                hi = std::max(hi, x);
            }
            uint16_t sb = f64_to_f16_bits((hi - lo) / 15.0);
            if ((sb & 0x7FFF) == 0x7C00) {
                err.bad = true;
                err.msg = "a group scale overflows fp16";
                return false;
            }
            if (hi == lo)
                sb = 0x3C00;  // 1.0
            else if (sb == 0)
                sb = 0x0001;  // 2^-24
            double s = f16_bits_to_f64(sb);
            // +0.0 turns a -0.0 zero point into the canonical +0
            double z = std::min(std::max(std::nearbyint(-lo / s), 0.0), 15.0) + 0.0;
            d.s[n * G + g] = sb;
            d.z[n * G + g] = f64_to_f16_bits(z);
            for (int j = 0; j < kGroup; ++j) {
                double x = static_cast<double>(v[j]);
                double c = std::min(std::max(std::nearbyint(x / s) + z, 0.0), 15.0);
                q[g * kGroup + j] = static_cast<uint8_t>(c);
                E[g * kGroup + j] = x - (c - z) * s;
            }
        }
    }
    return true;
}

// D4 for row n over its residual columns cols[0..cnt) (ascending), written
// at d.col/d.qr[base..base+cnt).
bool residual_row(const double *E, const int32_t *cols, int64_t cnt, int64_t n, int64_t base,
                  HostDecomp &d, RowError &err) {
    double a = 0.0;
    for (int64_t e = 0; e < cnt; ++e) a = std::max(a, std::fabs(E[cols[e]]));
    uint16_t srb = f64_to_f16_bits(a / 7.0);
    if ((srb & 0x7FFF) == 0x7C00) {
        err.bad = true;
        err.msg = "a residual scale overflows fp16";
        return false;
    }
    if (srb == 0) srb = 0x3C00;
    const double sr = f16_bits_to_f64(srb);
    d.sr[n] = srb;
    for (int64_t e = 0; e < cnt; ++e) {
        const int32_t c = cols[e];
        d.col[base + e] = c;
        d.qr[base + e] = static_cast<int8_t>(std::min(std::max(std::nearbyint(E[c] / sr), -8.0), 7.0));
    }
    return true;
}

// Row mode: decompose rows [r0, r1) of W into d (already sized).
void decompose_rows(const float *W, int64_t K, int64_t k_n, int64_t r0, int64_t r1,
                    HostDecomp &d, RowError &err) {
    std::vector<double> E(K), absE(K);
    std::vector<int32_t> idx(K);
    for (int64_t n = r0; n < r1; ++n) {
        if (!base_row(W, K, n, d, E.data(), err)) return;
        // residual: the k_n largest |E|, ties to the smaller column
        int64_t base = n * k_n;
        if (k_n > 0) {
            for (int64_t k = 0; k < K; ++k) absE[k] = std::fabs(E[k]);
            std::iota(idx.begin(), idx.end(), 0);
            auto before = [&](int32_t a, int32_t b) {
                return absE[a] > absE[b] || (absE[a] == absE[b] && a < b);
            };
            if (k_n < K) std::nth_element(idx.begin(), idx.begin() + k_n, idx.end(), before);
            std::sort(idx.begin(), idx.begin() + k_n);
            if (!residual_row(E.data(), idx.data(), k_n, n, base, d, err)) return;
        } else {
            d.sr[n] = 0x3C00;
        }
    }
}

// Block mode, pass 1: the base of the rows of row-blocks [b0, b1) and the
// delta score of each of their 16 x 64 blocks.
void score_blocks(const float *W, int64_t K, const float *h, int64_t b0, int64_t b1, HostDecomp &d,
                  std::vector<double> &score, RowError &err) {
    const int64_t nbc = K / kBlockCols;
    std::vector<double> E(kBlockRows * K);
    for (int64_t rb = b0; rb < b1; ++rb) {
        for (int r = 0; r < kBlockRows; ++r)
            if (!base_row(W, K, rb * kBlockRows + r, d, E.data() + r * K, err)) return;
        for (int64_t cb = 0; cb < nbc; ++cb) {
            double acc = 0.0;  // row by row, column by column
            for (int r = 0; r < kBlockRows; ++r)
                for (int c = 0; c < kBlockCols; ++c) {
                    const int64_t k = cb * kBlockCols + c;
                    const double e = E[r * K + k];
                    const double t = e * e;
                    const double w = h ? static_cast<double>(h[k]) : 1.0;
                    const double term = t * w;
                    acc = acc + term;
                }
            score[rb * nbc + cb] = acc;
        }
    }
}

// Block mode, pass 2: the residual of the rows of row-blocks [b0, b1) over
// the columns of their selected blocks (sel[rb * nbc + cb]).
void block_residual(const float *W, int64_t K, int64_t b0, int64_t b1, const std::vector<uint8_t> &sel,
                    HostDecomp &d, RowError &err) {
    const int64_t nbc = K / kBlockCols;
    std::vector<double> E(K);
    std::vector<int32_t> cols;
    for (int64_t rb = b0; rb < b1; ++rb) {
        cols.clear();
        for (int64_t cb = 0; cb < nbc; ++cb)
            if (sel[rb * nbc + cb])
                for (int c = 0; c < kBlockCols; ++c) cols.push_back(static_cast<int32_t>(cb * kBlockCols + c));
        for (int r = 0; r < kBlockRows; ++r) {
            const int64_t n = rb * kBlockRows + r;
            if (cols.empty()) {
                d.sr[n] = 0x3C00;
                continue;
            }
            if (!base_row(W, K, n, d, E.data(), err)) return;
            if (!residual_row(E.data(), cols.data(), static_cast<int64_t>(cols.size()), n, d.row_ptr[n], d,
                              err))
                return;
        }
    }
}

template <class F>
void parallel_rows(int64_t units, F &&body, std::vector<RowError> &errs) {
    unsigned hw = std::max(1u, std::thread::hardware_concurrency());
    int64_t nthreads = std::min<int64_t>(std::min<int64_t>(hw, 32), std::max<int64_t>(1, units / 4));
    errs.assign(nthreads, RowError());
    std::vector<std::thread> pool;
    int64_t chunk = (units + nthreads - 1) / nthreads;
    for (int64_t t = 0; t < nthreads; ++t) {
        int64_t u0 = t * chunk, u1 = std::min(units, u0 + chunk);
        if (u0 >= u1) continue;
        pool.emplace_back([&, t, u0, u1] { body(u0, u1, errs[t]); });
    }
    for (auto &th : pool) th.join();
}

mq_status decompose_blocks_host(const float *W, int64_t N, int64_t K, const mq_pack_opts &opts,
                                HostDecomp &d) {
    const int64_t G = K / kGroup, nbr = N / kBlockRows, nbc = K / kBlockCols;
    const int64_t nsel = residual_blocks_selected(N, K, opts.block_fraction);
    std::vector<double> score;
    std::vector<uint8_t> sel;
    try {
        d.q.assign(N * K, 0);
        d.s.assign(N * G, 0);
        d.z.assign(N * G, 0);
        d.row_ptr.assign(N + 1, 0);
        d.sr.assign(N, 0x3C00);
        score.assign(nbr * nbc, 0.0);
        sel.assign(nbr * nbc, 0);
    } catch (const std::bad_alloc &) {
        return fail(MQ_ERR_OUT_OF_MEMORY, "host allocation for the decomposition failed");
    }
    std::vector<RowError> errs;
    parallel_rows(nbr, [&](int64_t b0, int64_t b1, RowError &e) {
        score_blocks(W, K, opts.channel_weight, b0, b1, d, score, e);
    }, errs);
    for (auto &e : errs)
        if (e.bad) return fail(MQ_ERR_INVALID_ARG, e.msg);
    // the nsel largest scores, ties to the smaller block index
    std::vector<int64_t> order(nbr * nbc);
    std::iota(order.begin(), order.end(), int64_t(0));
    auto before = [&](int64_t a, int64_t b) { return score[a] > score[b] || (score[a] == score[b] && a < b); };
    if (nsel < nbr * nbc) std::nth_element(order.begin(), order.begin() + nsel, order.end(), before);
    for (int64_t i = 0; i < nsel; ++i) sel[order[i]] = 1;
    for (int64_t rb = 0; rb < nbr; ++rb) {
        int64_t cnt = 0;
        for (int64_t cb = 0; cb < nbc; ++cb) cnt += sel[rb * nbc + cb];
        for (int r = 0; r < kBlockRows; ++r) {
            const int64_t n = rb * kBlockRows + r;
            d.row_ptr[n + 1] = d.row_ptr[n] + cnt * kBlockCols;
        }
    }
    try {
        d.col.assign(d.row_ptr[N], 0);
        d.qr.assign(d.row_ptr[N], 0);
    } catch (const std::bad_alloc &) {
        return fail(MQ_ERR_OUT_OF_MEMORY, "host allocation for the decomposition failed");
    }
    parallel_rows(nbr, [&](int64_t b0, int64_t b1, RowError &e) { block_residual(W, K, b0, b1, sel, d, e); },
                  errs);
    for (auto &e : errs)
        if (e.bad) return fail(MQ_ERR_INVALID_ARG, e.msg);
    return MQ_OK;
}

}  // namespace

mq_status decompose_host(const float *W, int64_t N, int64_t K, const mq_pack_opts &opts, HostDecomp &d) {
    if (std::fegetround() != FE_TONEAREST)
        return fail(MQ_ERR_UNSUPPORTED, "the host FPU rounding mode must be round-to-nearest");
    d.N = N;
    d.K = K;
    if (opts.residual_blocks == 1) return decompose_blocks_host(W, N, K, opts, d);
    const double rho = opts.residual_density;
    const int64_t G = K / kGroup, k_n = residual_count(K, rho);
    try {
        d.q.assign(N * K, 0);
        d.s.assign(N * G, 0);
        d.z.assign(N * G, 0);
        d.row_ptr.resize(N + 1);
        d.col.assign(N * k_n, 0);
        d.qr.assign(N * k_n, 0);
        d.sr.assign(N, 0x3C00);
    } catch (const std::bad_alloc &) {
        return fail(MQ_ERR_OUT_OF_MEMORY, "host allocation for the decomposition failed");
    }
    for (int64_t n = 0; n <= N; ++n) d.row_ptr[n] = n * k_n;
    unsigned hw = std::max(1u, std::thread::hardware_concurrency());
    int64_t nthreads = std::min<int64_t>(std::min<int64_t>(hw, 32), std::max<int64_t>(1, N / 64));
    std::vector<RowError> errs(nthreads);
    std::vector<std::thread> pool;
    int64_t chunk = (N + nthreads - 1) / nthreads;
    for (int64_t t = 0; t < nthreads; ++t) {
        int64_t r0 = t * chunk, r1 = std::min(N, r0 + chunk);
        if (r0 >= r1) continue;
        pool.emplace_back(decompose_rows, W, K, k_n, r0, r1, std::ref(d), std::ref(errs[t]));
    }
    for (auto &th : pool) th.join();
    for (auto &e : errs)
        if (e.bad) return fail(MQ_ERR_INVALID_ARG, e.msg);
    return MQ_OK;
}

mq_decomp view_of(const HostDecomp &d) {
    mq_decomp v;
    v.N = d.N;
    v.K = d.K;
    v.q = d.q.data();
    v.s = d.s.data();
    v.z = d.z.data();
    v.row_ptr = d.row_ptr.data();
    v.col = d.col.data();
    v.qr = d.qr.data();
    v.sr = d.sr.data();
    return v;
}

mq_status validate_decomp(const mq_decomp *d) {
    if (!d) return fail(MQ_ERR_INVALID_ARG, "decomposition is NULL");
    mq_pack_opts o{kGroup, 0.0, 0, 0.0, nullptr};
    if (mq_status st = check_shape(d->N, d->K, &o)) return st;
    if (!d->q || !d->s || !d->z || !d->row_ptr || !d->sr)
        return fail(MQ_ERR_INVALID_ARG, "a decomposition array is NULL");
    const int64_t N = d->N, K = d->K, G = K / kGroup;
    if (d->row_ptr[0] != 0) return fail(MQ_ERR_INVALID_ARG, "row_ptr[0] must be 0");
    for (int64_t n = 0; n < N; ++n)
        if (d->row_ptr[n + 1] < d->row_ptr[n])
            return fail(MQ_ERR_INVALID_ARG, "row_ptr must be non-decreasing");
    const int64_t nnz = d->row_ptr[N];
    if (nnz > 0 && (!d->col || !d->qr)) return fail(MQ_ERR_INVALID_ARG, "col/qr are NULL");
    if (nnz >= (int64_t(1) << 31)) return fail(MQ_ERR_INVALID_ARG, "too many residual entries");
    for (int64_t i = 0; i < N * K; ++i)
        if (d->q[i] > 15) return fail(MQ_ERR_INVALID_ARG, "base code out of 0..15");
    for (int64_t i = 0; i < N * G; ++i) {
        double s = f16_bits_to_f64(d->s[i]), z = f16_bits_to_f64(d->z[i]);
        if (!std::isfinite(s)) return fail(MQ_ERR_INVALID_ARG, "non-finite group scale");
        if (!(z >= 0.0 && z <= 15.0 && z == std::floor(z)))
            return fail(MQ_ERR_INVALID_ARG, "zero point must be an integer 0..15");
    }
    for (int64_t n = 0; n < N; ++n) {
        if (!std::isfinite(f16_bits_to_f64(d->sr[n])))
            return fail(MQ_ERR_INVALID_ARG, "non-finite residual scale");
        for (int64_t e = d->row_ptr[n]; e < d->row_ptr[n + 1]; ++e) {
            if (d->col[e] < 0 || d->col[e] >= K)
                return fail(MQ_ERR_INVALID_ARG, "residual column out of range");
            if (e > d->row_ptr[n] && d->col[e] <= d->col[e - 1])
                return fail(MQ_ERR_INVALID_ARG, "residual columns must ascend within a row");
            if (d->qr[e] < -8 || d->qr[e] > 7)
                return fail(MQ_ERR_INVALID_ARG, "residual code out of -8..7");
        }
    }
    return MQ_OK;
}

bool block_tiles_host(const HostPacked &p, HostBlocks &b) {
    static const int kPi[8] = {0, 2, 4, 6, 1, 3, 5, 7};
    b = HostBlocks();
    const int64_t N = p.N, K = p.K;
    if (p.nnz == 0 || N % kBlockRows || K % kBlockCols) return false;
    const int64_t nbr = N / kBlockRows, nbc = K / kBlockCols;
    std::vector<int32_t> ptr(nbr + 1, 0);
    std::vector<uint16_t> cols;
    for (int64_t rb = 0; rb < nbr; ++rb) {
        const int64_t r0 = rb * kBlockRows;
        const int64_t len = p.row_ptr[r0 + 1] - p.row_ptr[r0];
        if (len % kBlockCols) return false;
        const int64_t nb = len / kBlockCols;
        for (int64_t r = r0; r < r0 + kBlockRows; ++r) {
            if (p.row_ptr[r + 1] - p.row_ptr[r] != len) return false;
            for (int64_t k = 0; k < nb; ++k) {
                const int64_t e = p.row_ptr[r] + k * kBlockCols;
                const int64_t c0 = p.col[e];
                if (c0 % kBlockCols) return false;
                if (r > r0 && c0 != p.col[p.row_ptr[r0] + k * kBlockCols]) return false;
                for (int64_t i = 1; i < kBlockCols; ++i)
                    if (p.col[e + i] != c0 + i) return false;
            }
        }
        for (int64_t k = 0; k < nb; ++k)
            cols.push_back(static_cast<uint16_t>(p.col[p.row_ptr[r0] + k * kBlockCols] / kBlockCols));
        ptr[rb + 1] = ptr[rb] + static_cast<int32_t>(nb);
    }
    b.nblk = static_cast<int64_t>(cols.size());
    b.map_words = (nbc + 31) / 32;
    b.ptr = std::move(ptr);
    b.col = std::move(cols);
    b.q.assign(b.nblk * kBlockRows * (kBlockCols / 8), 0);
    b.map.assign(nbr * b.map_words, 0);
    for (int64_t rb = 0; rb < nbr; ++rb)
        for (int64_t k = 0; k < b.ptr[rb + 1] - b.ptr[rb]; ++k) {
            const int64_t blk = b.ptr[rb] + k, cb = b.col[blk];
            b.map[rb * b.map_words + cb / 32] |= 1u << (cb % 32);
            for (int64_t r = 0; r < kBlockRows; ++r) {
                const int64_t e0 = p.row_ptr[rb * kBlockRows + r] + k * kBlockCols;
                for (int64_t w = 0; w < kBlockCols / 8; ++w) {
                    uint32_t word = 0;
                    for (int j = 0; j < 8; ++j) {
                        const int64_t e = e0 + 8 * w + kPi[j];
                        const uint32_t nib = (p.val[e >> 1] >> ((e & 1) * 4)) & 0xF;
                        word |= ((nib ^ 8u) & 0xF) << (4 * j);  // two's complement -> q_r + 8
                    }
                    b.q[(blk * kBlockRows + r) * (kBlockCols / 8) + w] = word;
                }
            }
        }
    return true;
}

void pack_host(const mq_decomp &d, HostPacked &p) {
    static const int kPi[8] = {0, 2, 4, 6, 1, 3, 5, 7};
    const int64_t N = d.N, K = d.K, G = K / kGroup;
    p.N = N;
    p.K = K;
    p.G = G;
    p.Gp = (G + 3) / 4 * 4;
    p.nnz = d.row_ptr[N];
    p.qweight.assign(N * (K / 8), 0);
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *q = d.q + n * K;
        uint32_t *out = p.qweight.data() + n * (K / 8);
        for (int64_t w = 0; w < K / 8; ++w) {
            uint32_t word = 0;
            for (int j = 0; j < 8; ++j) word |= uint32_t(q[8 * w + kPi[j]] & 0xF) << (4 * j);
            out[w] = word;
        }
    }
    p.sz.assign(N * p.Gp, 0);
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g)
            p.sz[n * p.Gp + g] = uint32_t(d.s[n * G + g]) | (uint32_t(d.z[n * G + g]) << 16);
    p.row_ptr.resize(N + 1);
    for (int64_t n = 0; n <= N; ++n) p.row_ptr[n] = static_cast<int32_t>(d.row_ptr[n]);
    p.col.resize(p.nnz);
    for (int64_t e = 0; e < p.nnz; ++e) p.col[e] = static_cast<uint16_t>(d.col[e]);
    p.val.assign((p.nnz + 1) / 2, 0);
    for (int64_t e = 0; e < p.nnz; ++e)
        p.val[e >> 1] |= uint8_t((uint8_t(d.qr[e]) & 0xF) << (4 * (e & 1)));
    p.rscale.assign(d.sr, d.sr + N);
}

}  // namespace mq
