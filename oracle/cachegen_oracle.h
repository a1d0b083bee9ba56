/*
 * cachegen_oracle.h -- TEST INFRASTRUCTURE ONLY: declarations of the plain CPU
 * oracle of the CacheGen codec (cachegen_oracle.c).  Used by the tests, the
 * smoke check and the benchmark's CPU baseline; never by the library.
 * Status returns: 0 ok, 1 invalid argument, 2 capacity, 3 corrupt,
 * 4 mismatch, 5 non-finite input.
 */
#ifndef CACHEGEN_ORACLE_H_
#define CACHEGEN_ORACLE_H_

#include <stdint.h>

float orc_f16_to_f32(uint16_t h);
uint16_t orc_f32_to_f16(float x);
void orc_f32_to_f16_array(const float* x, uint16_t* h, int64_t n);
void orc_f16_to_f32_array(const uint16_t* h, float* x, int64_t n);

int orc_layer_third(int l, int L);
float orc_step(int level, int l, int L);

void orc_anchor_params(const float* anchors, int m, float* zp, float* scale);
int orc_anchor_code(float x, float zp, float scale);
float orc_anchor_value(int c, float zp, float scale);
int orc_delta_code(float x, float ahat, float step);
float orc_delta_value(int q, float ahat, float step);

void orc_normalize(const uint32_t counts[255], uint64_t total, uint16_t f[256]);

/* One rANS stream over nsym symbols; symbol j uses freq[(j/per_table)*256 ..].
 * encode returns the number of u16 words written (negative on error). */
int64_t orc_rans_encode(const uint8_t* sym, int nsym, int per_table, const uint16_t* freq,
                        uint16_t* words, int64_t cap);
int orc_rans_decode(const uint16_t* words, int64_t nwords, int nsym, int per_table,
                    const uint16_t* freq, uint8_t* sym);

void orc_sections(int L, int H, int D, int64_t n, uint64_t offs[5]);
uint64_t orc_encoded_bound(int L, int H, int D, int C);

int orc_quantize_chunk(int L, int H, int D, const uint16_t* kv, int64_t T, int64_t token_start,
                       int C, int level, uint8_t* sym, float* zp, float* scale);
void orc_tables_of(int L, int H, int D, int64_t n, const uint8_t* sym, uint16_t* freq);
int orc_encode_chunk(int L, int H, int D, const uint16_t* kv, int64_t T, int64_t token_start,
                     int C, int level, uint8_t* out, uint64_t cap, uint64_t* out_size);
int orc_decode_chunk(const uint8_t* in, uint64_t in_bytes, int L, int H, int D, int C, int level,
                     uint16_t* out, uint64_t out_elems, int64_t* n_out, int64_t* start_out);

/* Format variants: adjacent = 0 is format 1 (deltas to the group's anchor);
 * adjacent = 1 is format 2 (deltas to the previous token's reconstruction,
 * header version 2).  The functions above are the adjacent = 0 forms. */
int orc_quantize_chunk_v(int L, int H, int D, const uint16_t* kv, int64_t T, int64_t token_start,
                         int C, int level, int adjacent, uint8_t* sym, float* zp, float* scale);
int orc_encode_chunk_v(int L, int H, int D, const uint16_t* kv, int64_t T, int64_t token_start,
                       int C, int level, int adjacent, uint8_t* out, uint64_t cap,
                       uint64_t* out_size);
int orc_decode_chunk_v(const uint8_t* in, uint64_t in_bytes, int L, int H, int D, int C,
                       int level, int adjacent, uint16_t* out, uint64_t out_elems,
                       int64_t* n_out, int64_t* start_out);

#endif
