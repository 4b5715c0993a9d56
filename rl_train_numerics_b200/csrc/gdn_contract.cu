// gdn_contract.cu -- identity digests of the CPR region's contract (host only).
//
// "NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI Training Runs",
// section "The execution contract": a contract pins every choice that can move
// bits and carries three SHA-256 identity digests -- semantic equivalence,
// numerical policy, and deployment settings that do not affect bits -- and two
// engines whose numerical policies differ refuse to run together.  Here the
// contract covers one region, this library's CPR Gated DeltaNet layer.  Each
// digest is the SHA-256 of a canonical text descriptor (the descriptor is
// exported too, so a peer can see what differs).
//
// The numerical-policy descriptor names the schedule versions below; any
// change to the arithmetic of the step, the boundary or the prep must bump
// the matching version, so that libraries with different bits cannot agree.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <string>

#include "../../include/gdn_cpr.h"

namespace {

// Schedule versions (part of the numerical policy).
constexpr int kStepSchedule = 2;      // per-token step: scaled mantissa, quad dots
constexpr int kBoundarySchedule = 3;  // boundary: prep (blocked T, scanned G) + walk
constexpr int kDescriptorFormat = 1;

// ---------------------------------------------------------------------------
// SHA-256 (FIPS 180-4): 512-bit blocks, 64 rounds of the compression function.
// ---------------------------------------------------------------------------
constexpr uint32_t kRound[64] = {
    0x428a2f98u, 0x71374491u, 0xb5c0fbcfu, 0xe9b5dba5u, 0x3956c25bu, 0x59f111f1u, 0x923f82a4u,
    0xab1c5ed5u, 0xd807aa98u, 0x12835b01u, 0x243185beu, 0x550c7dc3u, 0x72be5d74u, 0x80deb1feu,
    0x9bdc06a7u, 0xc19bf174u, 0xe49b69c1u, 0xefbe4786u, 0x0fc19dc6u, 0x240ca1ccu, 0x2de92c6fu,
    0x4a7484aau, 0x5cb0a9dcu, 0x76f988dau, 0x983e5152u, 0xa831c66du, 0xb00327c8u, 0xbf597fc7u,
    0xc6e00bf3u, 0xd5a79147u, 0x06ca6351u, 0x14292967u, 0x27b70a85u, 0x2e1b2138u, 0x4d2c6dfcu,
    0x53380d13u, 0x650a7354u, 0x766a0abbu, 0x81c2c92eu, 0x92722c85u, 0xa2bfe8a1u, 0xa81a664bu,
    0xc24b8b70u, 0xc76c51a3u, 0xd192e819u, 0xd6990624u, 0xf40e3585u, 0x106aa070u, 0x19a4c116u,
    0x1e376c08u, 0x2748774cu, 0x34b0bcb5u, 0x391c0cb3u, 0x4ed8aa4au, 0x5b9cca4fu, 0x682e6ff3u,
    0x748f82eeu, 0x78a5636fu, 0x84c87814u, 0x8cc70208u, 0x90befffau, 0xa4506cebu, 0xbef9a3f7u,
    0xc67178f2u};

inline uint32_t rotr(uint32_t x, int n) { return (x >> n) | (x << (32 - n)); }

void compress(uint32_t (&h)[8], const uint8_t* blk) {
  uint32_t w[64];
  for (int i = 0; i < 16; i++)
    w[i] = (uint32_t)blk[4 * i] << 24 | (uint32_t)blk[4 * i + 1] << 16 |
           (uint32_t)blk[4 * i + 2] << 8 | (uint32_t)blk[4 * i + 3];
  for (int i = 16; i < 64; i++) {
    const uint32_t s0 = rotr(w[i - 15], 7) ^ rotr(w[i - 15], 18) ^ (w[i - 15] >> 3);
    const uint32_t s1 = rotr(w[i - 2], 17) ^ rotr(w[i - 2], 19) ^ (w[i - 2] >> 10);
    w[i] = w[i - 16] + s0 + w[i - 7] + s1;
  }
  uint32_t a = h[0], b = h[1], c = h[2], d = h[3], e = h[4], f = h[5], g = h[6], hh = h[7];
  for (int i = 0; i < 64; i++) {
    const uint32_t t1 = hh + (rotr(e, 6) ^ rotr(e, 11) ^ rotr(e, 25)) + ((e & f) ^ (~e & g)) +
                        kRound[i] + w[i];
    const uint32_t t2 = (rotr(a, 2) ^ rotr(a, 13) ^ rotr(a, 22)) + ((a & b) ^ (a & c) ^ (b & c));
    hh = g;
    g = f;
    f = e;
    e = d + t1;
    d = c;
    c = b;
    b = a;
    a = t1 + t2;
  }
  h[0] += a;
  h[1] += b;
  h[2] += c;
  h[3] += d;
  h[4] += e;
  h[5] += f;
  h[6] += g;
  h[7] += hh;
}

void sha256(const uint8_t* data, size_t n, uint8_t out[32]) {
  uint32_t h[8] = {0x6a09e667u, 0xbb67ae85u, 0x3c6ef372u, 0xa54ff53au,
                   0x510e527fu, 0x9b05688cu, 0x1f83d9abu, 0x5be0cd19u};
  size_t i = 0;
  for (; i + 64 <= n; i += 64) compress(h, data + i);
  // Padding: 0x80, zeros, then the message length in bits (big endian).
  uint8_t tail[128] = {0};
  const size_t r = n - i;
  memcpy(tail, data + i, r);
  tail[r] = 0x80;
  const size_t tl = (r + 1 + 8 <= 64) ? 64 : 128;
  const uint64_t bits = (uint64_t)n * 8u;
  for (int k = 0; k < 8; k++) tail[tl - 1 - k] = (uint8_t)(bits >> (8 * k));
  compress(h, tail);
  if (tl == 128) compress(h, tail + 64);
  for (int k = 0; k < 8; k++)
    for (int b = 0; b < 4; b++) out[4 * k + b] = (uint8_t)(h[k] >> (24 - 8 * b));
}

const char* dtype_name(int d) { return d == GDN_BF16 ? "bf16" : "f32"; }

bool supported(int in_dtype, int out_dtype, int dk, int dv, int C) {
  if ((in_dtype != GDN_BF16 && in_dtype != GDN_F32) ||
      (out_dtype != GDN_BF16 && out_dtype != GDN_F32))
    return false;
  if (dk != dv || (dk != 64 && dk != 128) || C != 64) return false;
  return !(in_dtype == GDN_F32 && dk != 64);
}

std::string line(const char* key, const std::string& val) { return std::string(key) + "=" + val + "\n"; }
std::string num(long long v) { return std::to_string(v); }

// Canonical descriptor text: "key=value" lines in a fixed order.
std::string descriptor(int kind, int in_dtype, int out_dtype, int dk, int dv, int C) {
  std::string s = "gdn-cpr contract descriptor v" + num(kDescriptorFormat) + "\n";
  s += line("region", "cpr_gated_deltanet_forward_decode");
  if (kind == GDN_DIGEST_SEMANTIC) {
    s += line("digest", "semantic");
    s += line("recurrence", "S_t=exp(g_t)*S_{t-1}*(I-beta_t*k_t*k_t^T)+beta_t*v_t*k_t^T");
    s += line("output", "o_t=scale*S_t*q_t");
    s += line("state", "fp32[d_v][d_k], row=value channel");
    s += line("chunks", "C tokens from each sequence's token 0; boundary state every C tokens");
    s += line("gradients", "dL/d(q,k,v,beta,g,h0) of the recurrence given dL/do, dL/dS_final");
    s += line("d_k", num(dk));
    s += line("d_v", num(dv));
    s += line("C", num(C));
  } else if (kind == GDN_DIGEST_POLICY) {
    const bool tc = dk == 128 && in_dtype == GDN_BF16;
    s += line("digest", "numerical_policy");
    s += line("d_k", num(dk));
    s += line("d_v", num(dv));
    s += line("C", num(C));
    s += line("in_dtype", dtype_name(in_dtype));
    s += line("out_dtype", dtype_name(out_dtype));
    s += line("state_dtype", "f32");
    s += line("step_schedule", num(kStepSchedule));
    s += line("step",
              "scaled mantissa S=c*M, renormalise below 2^-64; per-row dots over a quad of "
              "lanes, 4 rows x 32 columns per lane in packed f32 pairs, xor butterfly 1,2; "
              "u=beta*fma(-a,c*p,v); o=(c*dot)*scale");
    s += line("boundary_schedule", num(kBoundarySchedule));
    s += line("prep",
              "P=KK^T mma.sync m16n8k16 bf16; G pair sums + Kogge-Stone scan (f64); T blocked "
              "16x16 forward substitution (f32)");
    s += line("walk", tc ? "tcgen05.mma kind::f16 M=128: Y n64, Z n(64-16ks), P n128; "
                           "A operands in tensor memory; S'=fma(exp(G_C),S,P)"
                         : "mma.sync m16n8k16 bf16, state in accumulator registers");
    s += line("splits", in_dtype == GDN_BF16 ? "state/Y/U 2 bf16 terms, Tb/Tv 2, K/V 1"
                                             : "state/Y/U 3 bf16 terms, Tb/Tv 3, K/V 3");
    s += line("backward",
              in_dtype == GDN_BF16
                  ? "boundary states by the forward's first pass; adjoint in chunk form "
                    "(prep: T, Pm, X; reverse walk over chunk ends; W = T^T R) by mma.sync "
                    "m16n8k16 bf16 with fp32 operands in 3 bf16 terms, all pairs of order < 3; "
                    "chunk u = T diag(beta)(V - diag(e^G) K S_a^T) by mma.sync (S_a 2 terms, "
                    "T and Z 3); chunk products Y,X,DQ,DK by mma.sync with w,S_a,mu_e,"
                    "-(B+B^T) in 2 bf16 terms and u,A in 3, all pairs of order < the finer "
                    "split; dbeta = w.v - e^G k.(W S_a) - sum A'X, dg by a telescoped sum "
                    "with do.o = q.dq"
                  : "boundary states by the forward's first pass; adjoint scan per row (4 "
                    "packed accumulators per lane, xor butterfly 1,2); chunk states by the "
                    "step schedule; chunk products Y,X,A,B,DQ,DK in f32 fma, fixed order; dg "
                    "by a telescoped sum");
    s += line("rounding", "round to nearest even, IEEE denormals, no contraction");
    s += line("compile", "sm_100a -O3 --fmad=false -ftz=false -prec-div=true -prec-sqrt=true");
  } else {
    int dev = -1, sms = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    else
      cudaGetLastError();  // no device: the count stays 0
    s += line("digest", "deployment");
    s += line("abi_version", num(GDN_CPR_ABI_VERSION));
    s += line("work_distribution",
              "persistent grids sized by occupancy x SM count; which block runs a unit "
              "does not change its bits");
    s += line("sm_count", num(sms));
  }
  return s;
}

int validate(int kind, int in_dtype, int out_dtype, int dk, int dv, int C) {
  if (kind != GDN_DIGEST_SEMANTIC && kind != GDN_DIGEST_POLICY && kind != GDN_DIGEST_DEPLOYMENT)
    return GDN_ERR_INVALID_ARG;
  return supported(in_dtype, out_dtype, dk, dv, C) ? GDN_OK : GDN_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

int gdn_cpr_contract_descriptor(int kind, int in_dtype, int out_dtype, int dk, int dv, int C,
                                char* buf, size_t buf_bytes, size_t* len_out) {
  const int rc = validate(kind, in_dtype, out_dtype, dk, dv, C);
  if (rc != GDN_OK) return rc;
  const std::string s = descriptor(kind, in_dtype, out_dtype, dk, dv, C);
  if (len_out) *len_out = s.size();
  if (!buf) return GDN_OK;  // size query
  if (buf_bytes < s.size() + 1) return GDN_ERR_INVALID_ARG;
  memcpy(buf, s.c_str(), s.size() + 1);
  return GDN_OK;
}

int gdn_cpr_contract_digest(int kind, int in_dtype, int out_dtype, int dk, int dv, int C,
                            uint8_t* out32) {
  if (!out32) return GDN_ERR_INVALID_ARG;
  const int rc = validate(kind, in_dtype, out_dtype, dk, dv, C);
  if (rc != GDN_OK) return rc;
  const std::string s = descriptor(kind, in_dtype, out_dtype, dk, dv, C);
  sha256(reinterpret_cast<const uint8_t*>(s.data()), s.size(), out32);
  return GDN_OK;
}

int gdn_cpr_contract_check(const uint8_t* peer_policy32, int in_dtype, int out_dtype, int dk,
                           int dv, int C) {
  if (!peer_policy32) return GDN_ERR_INVALID_ARG;
  uint8_t mine[32];
  const int rc = gdn_cpr_contract_digest(GDN_DIGEST_POLICY, in_dtype, out_dtype, dk, dv, C, mine);
  if (rc != GDN_OK) return rc;
  return memcmp(mine, peer_policy32, 32) == 0 ? GDN_OK : GDN_ERR_CONTRACT;
}

int gdn_sha256(const void* data, size_t n, uint8_t* out32) {
  if (!out32 || (!data && n)) return GDN_ERR_INVALID_ARG;
  sha256(static_cast<const uint8_t*>(data), n, out32);
  return GDN_OK;
}

}  // extern "C"
