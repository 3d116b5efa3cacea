/*
 * Paged decode attention: CPU oracle (test infrastructure only).
 *
 * This file is the slow, obviously correct reference that the CUDA path is
 * checked against. Only the tests, the smoke check and the benchmark's CPU
 * baseline use it; the library never calls it and shares no code with it.
 *
 * Everything is computed in double precision from the exactly converted
 * inputs. The half and bfloat16 decoders below are this file's own, written
 * from the IEEE 754 binary16 and bfloat16 bit layouts.
 *
 * Pool layout, restated here independently of the library:
 *   element (phys_block, kv_head, slot, d) of a pool sits at flat index
 *   ((phys_block * num_kv_heads + kv_head) * block_size + slot) * head_dim + d
 * Token t of sequence s lives at phys_block = block_tables[s][t / block_size],
 * slot = t % block_size.
 *
 * Functions and the passages they follow:
 *   oracle_paged_decode        - page "PagedAttention" (newikis), section
 *                                "Mathematical formulation": the causal
 *                                attention definition, written out two-pass.
 *   oracle_paged_decode_blockwise - page "PagedAttention Analysis"
 *                                (ryotta.opik.net), section 3 and its
 *                                block-table lookup pseudocode: walk the
 *                                logical blocks, look up the physical block,
 *                                update a running max / denominator / output.
 *   oracle_paged_decode_partitioned - the split-context variant: each
 *                                fixed-size partition of the context computed
 *                                alone, then combined by log-sum-exp weights.
 *                                The same online-softmax algebra as the
 *                                pseudocode above, applied to partitions.
 *   oracle_cache_append        - page "PagedAttention 논문 쉽게 읽기"
 *                                (iplexlaw.co.kr), section 2: a new token's
 *                                K/V are written into its slot.
 *   oracle_block_copy          - page "추론 엔진에서의 메모리 가상화"
 *                                (molayo1419.me), copy-on-write section: the
 *                                old block's contents are copied to the new.
 *   oracle_block_swap          - page "PagedAttention Analysis"
 *                                (ryotta.opik.net), section 6: a preempted
 *                                sequence's blocks are copied to blocks of a
 *                                separate (CPU) pool and back.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F32 = 0, ORACLE_F16 = 1, ORACLE_BF16 = 2 };

enum {
  ORACLE_OK = 0,
  ORACLE_EBADARG = -1,
  ORACLE_EBADBLOCK = -2, /* a block-table entry outside [0, num_blocks) */
  ORACLE_ENOMEM = -3,
};

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int f = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + f), e - 25); /* (1 + f/2^10) * 2^(e-15) */
  return sign ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double load_elem(const void *base, size_t idx, int dtype) {
  switch (dtype) {
  case ORACLE_F32:
    return (double)((const float *)base)[idx];
  case ORACLE_F16:
    return oracle_half_to_double(((const uint16_t *)base)[idx]);
  default:
    return oracle_bf16_to_double(((const uint16_t *)base)[idx]);
  }
}

static size_t pool_index(int phys, int kv_head, int slot, int d, int num_kv_heads,
                         int block_size, int head_dim) {
  return (((size_t)phys * num_kv_heads + kv_head) * block_size + slot) * head_dim + d;
}

static int check_args(int S, int Hq, int Hkv, int D, int B, int max_blocks, int dtype) {
  if (S < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || B <= 0 || max_blocks < 0) return ORACLE_EBADARG;
  if (Hq % Hkv != 0) return ORACLE_EBADARG;
  if (dtype < ORACLE_F32 || dtype > ORACLE_BF16) return ORACLE_EBADARG;
  return ORACLE_OK;
}

/*
 * Gather the first L tokens of one sequence and one KV head into contiguous
 * arrays k[L][D], v[L][D]. Returns ORACLE_EBADBLOCK on an out-of-range entry.
 */
static int gather_tokens(double *k, double *v, const void *k_pool, const void *v_pool,
                         const int32_t *table, int L, int kv_head, int Hkv, int D, int B,
                         int num_blocks, int max_blocks, int dtype) {
  for (int t = 0; t < L; ++t) {
    int j = t / B;
    if (j >= max_blocks) return ORACLE_EBADBLOCK;
    int phys = table[j];
    if (phys < 0 || phys >= num_blocks) return ORACLE_EBADBLOCK;
    for (int d = 0; d < D; ++d) {
      size_t idx = pool_index(phys, kv_head, t % B, d, Hkv, B, D);
      k[(size_t)t * D + d] = load_elem(k_pool, idx, dtype);
      v[(size_t)t * D + d] = load_elem(v_pool, idx, dtype);
    }
  }
  return ORACLE_OK;
}

/*
 * Attention of one query vector over L contiguous keys/values, written as the
 * definition: x_t = scale * q.k_t, a_t = exp(x_t - max) / sum exp(x_u - max),
 * o = sum a_t v_t. Also returns lse = max + ln(sum exp(x_t - max)) (natural log).
 * L == 0 gives o = 0 and lse = -inf.
 */
static void attend_contiguous(double *o, double *lse, const double *q, const double *k,
                              const double *v, int L, int D, double scale, double *x) {
  for (int d = 0; d < D; ++d) o[d] = 0.0;
  if (L <= 0) {
    *lse = -INFINITY;
    return;
  }
  double m = -INFINITY;
  for (int t = 0; t < L; ++t) {
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += q[d] * k[(size_t)t * D + d];
    x[t] = scale * dot;
    if (x[t] > m) m = x[t];
  }
  double denom = 0.0;
  for (int t = 0; t < L; ++t) {
    x[t] = exp(x[t] - m);
    denom += x[t];
  }
  for (int t = 0; t < L; ++t) {
    double a = x[t] / denom;
    for (int d = 0; d < D; ++d) o[d] += a * v[(size_t)t * D + d];
  }
  *lse = m + log(denom);
}

/*
 * out[S][Hq][D] (double) = attention of q[s][h] over the context_lens[s]
 * tokens of sequence s, read through its block table from KV head
 * h / (Hq / Hkv). lse_out (nullable) receives [S][Hq] natural-log
 * log-sum-exp values of the scaled scores.
 */
int oracle_paged_decode(double *out, double *lse_out, const void *q, const void *k_pool,
                        const void *v_pool, const int32_t *block_tables,
                        const int32_t *context_lens, int S, int Hq, int Hkv, int D, int B,
                        int max_blocks, int num_blocks, double scale, int dtype) {
  int rc = check_args(S, Hq, Hkv, D, B, max_blocks, dtype);
  if (rc) return rc;
  int G = Hq / Hkv;
  int status = ORACLE_OK;
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int s = 0; s < S; ++s) {
    for (int h = 0; h < Hq; ++h) {
      int L = context_lens[s] > 0 ? context_lens[s] : 0;
      size_t n = (size_t)(L > 0 ? L : 1);
      double *k = malloc(n * D * sizeof(double));
      double *v = malloc(n * D * sizeof(double));
      double *x = malloc(n * sizeof(double));
      double *qd = malloc((size_t)D * sizeof(double));
      double *o = out + ((size_t)s * Hq + h) * D;
      double lse;
      if (!k || !v || !x || !qd) {
#pragma omp atomic write
        status = ORACLE_ENOMEM;
      } else {
        for (int d = 0; d < D; ++d) qd[d] = load_elem(q, ((size_t)s * Hq + h) * D + d, dtype);
        int r = gather_tokens(k, v, k_pool, v_pool, block_tables + (size_t)s * max_blocks, L,
                              h / G, Hkv, D, B, num_blocks, max_blocks, dtype);
        if (r) {
#pragma omp atomic write
          status = r;
        } else {
          attend_contiguous(o, &lse, qd, k, v, L, D, scale, x);
          if (lse_out) lse_out[(size_t)s * Hq + h] = lse;
        }
      }
      free(k);
      free(v);
      free(x);
      free(qd);
    }
  }
  return status;
}

/*
 * The block-by-block form: for each logical block j the physical block is
 * looked up, the block's scores s = scale * q.K_j are formed, and a running
 * (max m, denominator l, unnormalised output acc) is updated:
 *   m' = max(m, max_t s_t)
 *   l' = l * exp(m - m') + sum_t exp(s_t - m')
 *   acc' = acc * exp(m - m') + sum_t exp(s_t - m') v_t
 * and o = acc / l after the last block. Only slots t < context_len count.
 */
int oracle_paged_decode_blockwise(double *out, const void *q, const void *k_pool,
                                  const void *v_pool, const int32_t *block_tables,
                                  const int32_t *context_lens, int S, int Hq, int Hkv, int D,
                                  int B, int max_blocks, int num_blocks, double scale,
                                  int dtype) {
  int rc = check_args(S, Hq, Hkv, D, B, max_blocks, dtype);
  if (rc) return rc;
  int G = Hq / Hkv;
  int status = ORACLE_OK;
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int s = 0; s < S; ++s) {
    for (int h = 0; h < Hq; ++h) {
      int L = context_lens[s] > 0 ? context_lens[s] : 0;
      int g = h / G;
      double *o = out + ((size_t)s * Hq + h) * D;
      double *qd = malloc((size_t)D * sizeof(double));
      double *acc = calloc((size_t)D, sizeof(double));
      double *sc = malloc((size_t)B * sizeof(double));
      if (!qd || !acc || !sc) {
#pragma omp atomic write
        status = ORACLE_ENOMEM;
        free(qd);
        free(acc);
        free(sc);
        continue;
      }
      for (int d = 0; d < D; ++d) qd[d] = load_elem(q, ((size_t)s * Hq + h) * D + d, dtype);
      double m = -INFINITY, l = 0.0;
      int nblocks = (L + B - 1) / B;
      int bad = 0;
      for (int j = 0; j < nblocks && !bad; ++j) {
        int phys = j < max_blocks ? block_tables[(size_t)s * max_blocks + j] : -1;
        if (phys < 0 || phys >= num_blocks) {
          bad = 1;
          break;
        }
        int valid = L - j * B < B ? L - j * B : B;
        double bmax = -INFINITY;
        for (int t = 0; t < valid; ++t) {
          double dot = 0.0;
          for (int d = 0; d < D; ++d)
            dot += qd[d] * load_elem(k_pool, pool_index(phys, g, t, d, Hkv, B, D), dtype);
          sc[t] = scale * dot;
          if (sc[t] > bmax) bmax = sc[t];
        }
        double mn = m > bmax ? m : bmax;
        double alpha = exp(m - mn); /* m = -inf on the first block gives 0 */
        l *= alpha;
        for (int d = 0; d < D; ++d) acc[d] *= alpha;
        for (int t = 0; t < valid; ++t) {
          double p = exp(sc[t] - mn);
          l += p;
          for (int d = 0; d < D; ++d)
            acc[d] += p * load_elem(v_pool, pool_index(phys, g, t, d, Hkv, B, D), dtype);
        }
        m = mn;
      }
      if (bad) {
#pragma omp atomic write
        status = ORACLE_EBADBLOCK;
      } else {
        for (int d = 0; d < D; ++d) o[d] = L > 0 ? acc[d] / l : 0.0;
      }
      free(qd);
      free(acc);
      free(sc);
    }
  }
  return status;
}

/*
 * Split-context form: the context of each sequence is cut into partitions of
 * partition_size tokens. Each partition p gives its own normalised output o_p
 * and lse_p (natural log, as in attend_contiguous). The partitions are
 * combined as lse = log sum_p exp(lse_p) and o = sum_p exp(lse_p - lse) o_p.
 * part_o / part_lse (nullable) receive the per-partition values,
 * [S][Hq][max_parts][D] and [S][Hq][max_parts], with unused partitions left
 * at 0 / -inf.
 */
int oracle_paged_decode_partitioned(double *out, double *part_o, double *part_lse,
                                    int max_parts, const void *q, const void *k_pool,
                                    const void *v_pool, const int32_t *block_tables,
                                    const int32_t *context_lens, int S, int Hq, int Hkv, int D,
                                    int B, int max_blocks, int num_blocks, double scale,
                                    int dtype, int partition_size) {
  int rc = check_args(S, Hq, Hkv, D, B, max_blocks, dtype);
  if (rc) return rc;
  if (partition_size <= 0 || max_parts <= 0) return ORACLE_EBADARG;
  int G = Hq / Hkv;
  int status = ORACLE_OK;
  for (int s = 0; s < S; ++s) {
    int L = context_lens[s] > 0 ? context_lens[s] : 0;
    if ((L + partition_size - 1) / partition_size > max_parts) return ORACLE_EBADARG;
  }
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int s = 0; s < S; ++s) {
    for (int h = 0; h < Hq; ++h) {
      int L = context_lens[s] > 0 ? context_lens[s] : 0;
      int nparts = (L + partition_size - 1) / partition_size;
      size_t n = (size_t)(L > 0 ? L : 1);
      double *k = malloc(n * D * sizeof(double));
      double *v = malloc(n * D * sizeof(double));
      double *x = malloc(n * sizeof(double));
      double *qd = malloc((size_t)D * sizeof(double));
      double *po = malloc((size_t)(nparts > 0 ? nparts : 1) * D * sizeof(double));
      double *pl = malloc((size_t)(nparts > 0 ? nparts : 1) * sizeof(double));
      double *o = out + ((size_t)s * Hq + h) * D;
      if (!k || !v || !x || !qd || !po || !pl) {
#pragma omp atomic write
        status = ORACLE_ENOMEM;
      } else {
        for (int d = 0; d < D; ++d) qd[d] = load_elem(q, ((size_t)s * Hq + h) * D + d, dtype);
        int r = gather_tokens(k, v, k_pool, v_pool, block_tables + (size_t)s * max_blocks, L,
                              h / G, Hkv, D, B, num_blocks, max_blocks, dtype);
        if (r) {
#pragma omp atomic write
          status = r;
        } else {
          for (int p = 0; p < nparts; ++p) {
            int t0 = p * partition_size;
            int len = L - t0 < partition_size ? L - t0 : partition_size;
            attend_contiguous(po + (size_t)p * D, pl + p, qd, k + (size_t)t0 * D,
                              v + (size_t)t0 * D, len, D, scale, x);
          }
          double mx = -INFINITY;
          for (int p = 0; p < nparts; ++p)
            if (pl[p] > mx) mx = pl[p];
          double wsum = 0.0;
          for (int p = 0; p < nparts; ++p) wsum += exp(pl[p] - mx);
          double lse = mx + log(wsum);
          for (int d = 0; d < D; ++d) o[d] = 0.0;
          for (int p = 0; p < nparts; ++p) {
            double w = exp(pl[p] - lse);
            for (int d = 0; d < D; ++d) o[d] += w * po[(size_t)p * D + d];
          }
          if (part_o || part_lse) {
            for (int p = 0; p < max_parts; ++p) {
              size_t base = ((size_t)s * Hq + h) * max_parts + p;
              if (part_lse) part_lse[base] = p < nparts ? pl[p] : -INFINITY;
              if (part_o)
                for (int d = 0; d < D; ++d)
                  part_o[base * D + d] = p < nparts ? po[(size_t)p * D + d] : 0.0;
            }
          }
        }
      }
      free(k);
      free(v);
      free(x);
      free(qd);
      free(po);
      free(pl);
    }
  }
  return status;
}

/*
 * Cache append: for every token i with slot = slot_mapping[i] >= 0, copy the
 * D elements of k_new[i][h] and v_new[i][h] into pool slot (slot / B, slot % B)
 * of KV head h, for all heads. Negative slots are skipped. A slot at or
 * beyond num_blocks * B is an error (nothing is written for it).
 */
int oracle_cache_append(void *k_pool, void *v_pool, const void *k_new, const void *v_new,
                        const int64_t *slot_mapping, int num_tokens, int Hkv, int D, int B,
                        int num_blocks, int elem_bytes) {
  if (num_tokens < 0 || Hkv <= 0 || D <= 0 || B <= 0 || num_blocks < 0 || elem_bytes <= 0)
    return ORACLE_EBADARG;
  int status = ORACLE_OK;
  size_t row = (size_t)D * elem_bytes;
  for (int i = 0; i < num_tokens; ++i) {
    int64_t slot = slot_mapping[i];
    if (slot < 0) continue;
    if (slot >= (int64_t)num_blocks * B) {
      status = ORACLE_EBADBLOCK;
      continue;
    }
    int phys = (int)(slot / B), off = (int)(slot % B);
    for (int h = 0; h < Hkv; ++h) {
      size_t dst = pool_index(phys, h, off, 0, Hkv, B, D) * elem_bytes;
      size_t src = ((size_t)i * Hkv + h) * row;
      memcpy((char *)k_pool + dst, (const char *)k_new + src, row);
      memcpy((char *)v_pool + dst, (const char *)v_new + src, row);
    }
  }
  return status;
}

/*
 * Block copy: for each pair (src, dst), the whole physical block (all KV
 * heads, all B slots, all D elements) of both pools is copied src -> dst.
 * Pairs run in order. Out-of-range ids are an error, and that pair is skipped.
 */
int oracle_block_copy(void *k_pool, void *v_pool, const int32_t *pairs, int num_pairs, int Hkv,
                      int D, int B, int num_blocks, int elem_bytes) {
  if (num_pairs < 0 || Hkv <= 0 || D <= 0 || B <= 0 || elem_bytes <= 0) return ORACLE_EBADARG;
  int status = ORACLE_OK;
  size_t block_bytes = (size_t)Hkv * B * D * elem_bytes;
  for (int i = 0; i < num_pairs; ++i) {
    int src = pairs[2 * i], dst = pairs[2 * i + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      status = ORACLE_EBADBLOCK;
      continue;
    }
    memcpy((char *)k_pool + (size_t)dst * block_bytes, (const char *)k_pool + (size_t)src * block_bytes,
           block_bytes);
    memcpy((char *)v_pool + (size_t)dst * block_bytes, (const char *)v_pool + (size_t)src * block_bytes,
           block_bytes);
  }
  return status;
}

/*
 * Block swap: for each pair (src, dst), the whole block src of the source
 * pools is copied into block dst of the destination pools (both K and V).
 * Out-of-range ids (src against src_blocks, dst against dst_blocks) are an
 * error, and that pair is skipped.
 */
int oracle_block_swap(void *dst_k, void *dst_v, const void *src_k, const void *src_v,
                      const int32_t *pairs, int num_pairs, int Hkv, int D, int B,
                      int src_blocks, int dst_blocks, int elem_bytes) {
  if (num_pairs < 0 || Hkv <= 0 || D <= 0 || B <= 0 || elem_bytes <= 0) return ORACLE_EBADARG;
  int status = ORACLE_OK;
  size_t block_bytes = (size_t)Hkv * B * D * elem_bytes;
  for (int i = 0; i < num_pairs; ++i) {
    int src = pairs[2 * i], dst = pairs[2 * i + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
      status = ORACLE_EBADBLOCK;
      continue;
    }
    memcpy((char *)dst_k + (size_t)dst * block_bytes, (const char *)src_k + (size_t)src * block_bytes,
           block_bytes);
    memcpy((char *)dst_v + (size_t)dst * block_bytes, (const char *)src_v + (size_t)src * block_bytes,
           block_bytes);
  }
  return status;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
