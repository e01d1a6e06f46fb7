/*
 * synth_host.c - host entry points of the seeded input generator, for the
 * Python test and bench harness (ctypes).  Fills caller-owned host buffers.
 * No decoder arithmetic lives here.
 */
#include "synth.h"

void syn_fill_bf16_normal(uint64_t seed, uint32_t kind, uint32_t layer, uint32_t expert,
                          uint64_t start, uint64_t n, double sigma, uint16_t* out) {
  uint64_t key = syn_key(seed, syn_stream(kind, layer, expert));
  float sc = syn_normal_scale(sigma);
  for (uint64_t i = 0; i < n; ++i) out[i] = syn_bf16_normal(key, start + i, sc);
}

void syn_fill_bf16_gain(uint64_t seed, uint32_t kind, uint32_t layer, uint64_t n,
                        double sigma, uint16_t* out) {
  uint64_t key = syn_key(seed, syn_stream(kind, layer, 0));
  float sc = syn_normal_scale(sigma);
  for (uint64_t i = 0; i < n; ++i) out[i] = syn_bf16_gain(key, i, sc);
}

void syn_fill_e4m3_normal(uint64_t seed, uint32_t kind, uint32_t layer, uint32_t expert,
                          uint64_t start, uint64_t n, uint8_t* out) {
  uint64_t key = syn_key(seed, syn_stream(kind, layer, expert));
  float sc = syn_normal_scale(16.0);
  for (uint64_t i = 0; i < n; ++i) out[i] = syn_e4m3_normal(key, start + i, sc);
}

void syn_fill_block_scales(uint64_t seed, uint32_t kind, uint32_t layer, uint32_t expert,
                           uint64_t n, float base, float* out) {
  uint64_t key = syn_key(seed, syn_stream(SYN_FP8_SCALE, layer, (kind << 12) | expert));
  for (uint64_t i = 0; i < n; ++i) out[i] = syn_block_scale(key, i, base);
}

void syn_fill_tokens(uint64_t seed, uint32_t kind, uint64_t start, uint64_t n, uint32_t V,
                     int32_t* out) {
  uint64_t key = syn_key(seed, syn_stream(kind, 0, 0));
  for (uint64_t i = 0; i < n; ++i) out[i] = syn_token(key, start + i, V);
}

uint8_t syn_e4m3_encode(float f) { return syn_e4m3_rne(f); }
uint16_t syn_bf16_encode(float f) { return syn_bf16_rne(f); }
uint64_t syn_raw_u64(uint64_t seed, uint32_t kind, uint32_t layer, uint32_t expert, uint64_t i) {
  return syn_u64(syn_key(seed, syn_stream(kind, layer, expert)), i);
}
