// identity.cu -- contract identities of the CPR Gated DeltaNet layer (host code).
//
// The runtimes that must agree bit for bit (rollout prefill, decode, trainer
// forward) compare SHA-256 identities of the contract they execute, split into
// a semantic identity (what the layer computes), a numerical-policy identity
// (the arithmetic schedule: reduction trees, operation order, split products,
// instruction shapes) and a deployment identity (the build that runs it):
// IsoExec summary page, section "Contract Structure and Enforcement"
// (Identities); commentary blog, section 6 (why the contract gets a digest).
//
// Each identity is the SHA-256 (FIPS 180-4) of a canonical text that this file
// writes out; gdn_contract_text returns the text, so a caller can check the
// digest with any SHA-256 implementation.
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "gdn_cpr.h"

#ifndef GDN_SOURCES_SHA256
#define GDN_SOURCES_SHA256 "unknown"
#endif

namespace {

// ------------------------------------------------------------------ SHA-256
// FIPS 180-4, section 6.2: 64 rounds over 512-bit blocks; the round constants
// are the first 32 bits of the fractional parts of the cube roots of the first
// 64 primes, the initial hash those of the square roots of the first 8 primes
// (section 4.2.2 and 5.3.3).  They are derived here rather than tabulated.
struct Sha256Consts {
    uint32_t k[64];
    uint32_t h0[8];
};

// floor(frac(p^(1/r)) * 2^32) for r in {2, 3}: the low 32 bits of the largest
// integer x with x^r <= p * 2^(32 r), found bit by bit in exact 128-bit
// arithmetic (p <= 311, so x < 2^35 and x^3 < 2^105).
uint32_t frac_root_bits(uint32_t p, int r)
{
    const unsigned __int128 target = (unsigned __int128)p << (32 * r);
    unsigned __int128 x = 0;
    for (int bit = 34; bit >= 0; --bit) {
        const unsigned __int128 t = x | ((unsigned __int128)1 << bit);
        const unsigned __int128 pw = r == 2 ? t * t : t * t * t;
        if (pw <= target) x = t;
    }
    return (uint32_t)(x & 0xffffffffu);
}

const Sha256Consts& consts()
{
    static const Sha256Consts c = [] {
        Sha256Consts s{};
        uint32_t primes[64];
        int np = 0;
        for (uint32_t v = 2; np < 64; ++v) {
            bool prime = true;
            for (uint32_t d = 2; d * d <= v; ++d)
                if (v % d == 0) { prime = false; break; }
            if (prime) primes[np++] = v;
        }
        for (int i = 0; i < 64; ++i) s.k[i] = frac_root_bits(primes[i], 3);
        for (int i = 0; i < 8; ++i) s.h0[i] = frac_root_bits(primes[i], 2);
        return s;
    }();
    return c;
}

inline uint32_t rotr(uint32_t x, int n) { return (x >> n) | (x << (32 - n)); }

void sha256_block(uint32_t (&h)[8], const uint8_t* blk)
{
    const Sha256Consts& c = consts();
    uint32_t w[64];
    for (int t = 0; t < 16; ++t)
        w[t] = (uint32_t)blk[4 * t] << 24 | (uint32_t)blk[4 * t + 1] << 16 | (uint32_t)blk[4 * t + 2] << 8 |
               (uint32_t)blk[4 * t + 3];
    for (int t = 16; t < 64; ++t) {
        const uint32_t s0 = rotr(w[t - 15], 7) ^ rotr(w[t - 15], 18) ^ (w[t - 15] >> 3);
        const uint32_t s1 = rotr(w[t - 2], 17) ^ rotr(w[t - 2], 19) ^ (w[t - 2] >> 10);
        w[t] = w[t - 16] + s0 + w[t - 7] + s1;
    }
    uint32_t a = h[0], b = h[1], cc = h[2], d = h[3], e = h[4], f = h[5], g = h[6], hh = h[7];
    for (int t = 0; t < 64; ++t) {
        const uint32_t S1 = rotr(e, 6) ^ rotr(e, 11) ^ rotr(e, 25);
        const uint32_t ch = (e & f) ^ (~e & g);
        const uint32_t t1 = hh + S1 + ch + c.k[t] + w[t];
        const uint32_t S0 = rotr(a, 2) ^ rotr(a, 13) ^ rotr(a, 22);
        const uint32_t maj = (a & b) ^ (a & cc) ^ (b & cc);
        const uint32_t t2 = S0 + maj;
        hh = g; g = f; f = e; e = d + t1; d = cc; cc = b; b = a; a = t1 + t2;
    }
    h[0] += a; h[1] += b; h[2] += cc; h[3] += d; h[4] += e; h[5] += f; h[6] += g; h[7] += hh;
}

void sha256_hex(const uint8_t* data, size_t n, char* out)
{
    uint32_t h[8];
    std::memcpy(h, consts().h0, sizeof(h));
    size_t i = 0;
    for (; i + 64 <= n; i += 64) sha256_block(h, data + i);
    // padding: 0x80, zeros, then the message length in bits (64-bit big endian)
    uint8_t tail[128] = {0};
    const size_t rem = n - i;
    std::memcpy(tail, data + i, rem);
    tail[rem] = 0x80;
    const size_t tlen = rem < 56 ? 64 : 128;
    const uint64_t bits = (uint64_t)n * 8;
    for (int b = 0; b < 8; ++b) tail[tlen - 1 - b] = (uint8_t)(bits >> (8 * b));
    for (size_t o = 0; o < tlen; o += 64) sha256_block(h, tail + o);
    static const char* hex = "0123456789abcdef";
    for (int w = 0; w < 8; ++w)
        for (int b = 0; b < 4; ++b) {
            const uint8_t byte = (uint8_t)(h[w] >> (24 - 8 * b));
            out[8 * w + 2 * b] = hex[byte >> 4];
            out[8 * w + 2 * b + 1] = hex[byte & 15];
        }
    out[64] = '\0';
}

// ------------------------------------------------------------------ texts
bool shape_ok(int32_t d_k, int32_t d_v, int32_t C, gdn_dtype_t in_dtype, gdn_dtype_t out_dtype)
{
    const bool d_ok = d_k == d_v && (d_k == 16 || d_k == 32 || d_k == 64 || d_k == 128);
    const bool c_ok = C == 16 || C == 32 || C == 64;
    const bool t_ok = (in_dtype == GDN_F32 || in_dtype == GDN_BF16) && (out_dtype == GDN_F32 || out_dtype == GDN_BF16);
    return d_ok && c_ok && t_ok;
}

const char* dtype_name(gdn_dtype_t t) { return t == GDN_BF16 ? "bf16" : "f32"; }

const char* kSemantic =
    "gated-deltanet-cpr semantic identity\n"
    "recurrence: S_t = alpha_t * S_{t-1} * (I - beta_t * k_t * k_t^T) + beta_t * v_t * k_t^T; o_t = S_t * q_t\n"
    "state: fp32 [d_v][d_k]; state_in is the state at each sequence's position 0 (zeros when absent)\n"
    "chunking: boundaries every C tokens from each sequence's own token 0\n"
    "composition: boundary states by the chunk update P_chunk; every output by the per-token recurrence P_tok\n"
    "  started at its chunk's boundary state; decode runs P_tok and after C buffered tokens sets\n"
    "  S_b <- P_chunk(S_b, buffer), and the running state <- S_b\n"
    "inputs: q, k [T][H][d_k], v [T][H][d_v] in in_dtype (bf16 widened exactly); alpha, beta [T][H] fp32; no q scaling\n"
    "outputs: o [T][H][d_v] in out_dtype; chunk states at positions 0, C, ..., floor(L/C)*C\n";

const char* kPolicy =
    "gated-deltanet-cpr numerical policy identity\n"
    "fp32 operations: IEEE binary32, round to nearest even, subnormals kept, no contraction\n"
    "tree(x, y): 8 leaves of d_k/8 contiguous elements; leaf = x[0]*y[0], then fma ascending;\n"
    "  result ((l0+l1)+(l2+l3))+((l4+l5)+(l6+l7))\n"
    "P_tok on a running state c*R (c = 1, R = the boundary state at a chunk start), per token:\n"
    "  kq = tree(k, q); cn = alpha*c; per row i, over R before the token: dk = tree(R_i, k), dq = tree(R_i, q),\n"
    "  d = beta*(v_i - cn*dk); if cn >= 2^-64: dt = d*rcp.rn(cn), R_ij = fma(dt, k_j, R_ij),\n"
    "  o_i = cn*fma(dt, kq, dq), c = cn; else (fold): R_ij = fma(d, k_j, cn*R_ij), o_i = fma(d, kq, cn*dq), c = 1\n"
    "split of an fp32 operand x: hi = cvt.rna.tf32(x), lo = cvt.rna.tf32(x - hi); k has no lo part for bf16 inputs\n"
    "P_chunk part 1: decays D[s][s] = 1, D[t][s] = D[t-1][s]*alpha_t;\n"
    "  Gram G[t][s] = k_t.k_s (s < t) by mma.sync.m16n8k8 tf32, fp32 accumulate, K blocks of 8 ascending:\n"
    "  bf16 inputs: four accumulators by K block mod 4, G = (a0+a1)+(a2+a3); else G = (lo.hi + hi.lo) + hi.hi;\n"
    "  A[t][s] = beta_t*(D[t][s]*G[t][s]) (s < t); T = (I + A)^-1 in blocks of 16 tokens:\n"
    "  diagonal blocks by substitution, T[i][i] = 1, T[t][i] = fma chain over s = i..t-1 ascending of\n"
    "  (-A[t][s])*T[s][i] from 0; block (i, j < i) by distance i - j ascending: M = A[i][j..i-1] T[j..i-1][j],\n"
    "  T[i][j] = -(T[i][i] M), both by mma.sync.m16n8k8 tf32 split products (lo.hi + hi.lo) + hi.hi;\n"
    "  gamma_t = beta_t*D[t][0]; u0 = (T diag(beta)) V, w = (T diag(gamma)) K by mma.sync.m16n8k8 tf32,\n"
    "  row block r over K blocks 0..2r+1 ascending: bf16 inputs (V, K exact) lo.V + hi.V,\n"
    "  else (lo.hi + hi.lo) + hi.hi\n"
    "P_chunk part 2: tcgen05.mma kind::tf32, M = 128, A in tensor memory, B K-major in shared memory,\n"
    "  fp32 accumulate, one accumulator per phase fed in this order: lo.hi over K blocks of 8 ascending,\n"
    "  then hi.lo, then hi.hi;\n"
    "  E = S_lo.w_hi ; S_hi.w_lo ; S_hi.w_hi (one accumulator);\n"
    "  e_t = D[C][t]*(u0_t - E);\n"
    "  P = e_lo.k_hi [; e_hi.k_lo] ; e_hi.k_hi (one accumulator), the bracket absent for bf16 inputs;\n"
    "  S' = D[C][0]*S + P\n"
    "output store: fp32, or bf16 round to nearest even\n";

int write_text(gdn_identity_kind_t kind, int32_t d_k, int32_t d_v, int32_t C, gdn_dtype_t in_dtype,
               gdn_dtype_t out_dtype, char* buf, size_t cap)
{
    const char* ind = dtype_name(in_dtype);
    const char* outd = dtype_name(out_dtype);
    switch (kind) {
    case GDN_ID_SEMANTIC:
        return std::snprintf(buf, cap, "%sd_k=%d d_v=%d C=%d in=%s out=%s\n", kSemantic, d_k, d_v, C, ind, outd);
    case GDN_ID_NUMERICAL_POLICY:
        return std::snprintf(buf, cap, "%scontract=%s\nd_k=%d d_v=%d C=%d in=%s out=%s\n", kPolicy,
                             gdn_contract_id(), d_k, d_v, C, ind, outd);
    case GDN_ID_DEPLOYMENT:
        return std::snprintf(buf, cap,
                             "gated-deltanet-cpr deployment identity\ntarget=sm_100a\nkernel_sources_sha256=%s\n"
                             "nvcc=%d.%d.%d\ncontract=%s\nd_k=%d d_v=%d C=%d in=%s out=%s\n",
                             GDN_SOURCES_SHA256, __CUDACC_VER_MAJOR__, __CUDACC_VER_MINOR__,
                             __CUDACC_VER_BUILD__, gdn_contract_id(), d_k, d_v, C, ind, outd);
    }
    return -1;
}

}  // namespace

extern "C" {

gdn_status_t gdn_sha256_hex(const void* data, size_t n, char* out_hex)
{
    if (out_hex == nullptr || (data == nullptr && n != 0)) return GDN_ERR_INVALID_ARG;
    sha256_hex(static_cast<const uint8_t*>(data), n, out_hex);
    return GDN_OK;
}

int64_t gdn_contract_text(gdn_identity_kind_t kind, int32_t d_k, int32_t d_v, int32_t C, gdn_dtype_t in_dtype,
                          gdn_dtype_t out_dtype, char* buf, size_t cap)
{
    if (!shape_ok(d_k, d_v, C, in_dtype, out_dtype)) return -1;
    if (buf == nullptr && cap != 0) return -1;
    char dummy[1];
    const int n = write_text(kind, d_k, d_v, C, in_dtype, out_dtype, cap ? buf : dummy, cap ? cap : 1);
    return n < 0 ? -1 : (int64_t)n;
}

gdn_status_t gdn_contract_identity(gdn_identity_kind_t kind, int32_t d_k, int32_t d_v, int32_t C,
                                   gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, char* out_hex)
{
    if (out_hex == nullptr) return GDN_ERR_INVALID_ARG;
    if (!shape_ok(d_k, d_v, C, in_dtype, out_dtype)) return GDN_ERR_UNSUPPORTED;
    char buf[8192];
    const int n = write_text(kind, d_k, d_v, C, in_dtype, out_dtype, buf, sizeof(buf));
    if (n < 0 || (size_t)n >= sizeof(buf)) return GDN_ERR_INVALID_ARG;
    sha256_hex(reinterpret_cast<const uint8_t*>(buf), (size_t)n, out_hex);
    return GDN_OK;
}

}  // extern "C"
