/*
 * A plain-C caller of libkvq (include/kvq.h): no PyTorch, device buffers
 * from cudaMalloc, sizes from the library's own sizing calls.  It fills an
 * INT4 G64 cache of 2 sequences x 2 KV heads with 300 tokens by one bulk
 * kvq_quantize_append, gives the sequences ragged lengths, runs
 * kvq_decode_attention for 4 query heads per KV head, and writes its inputs
 * and every output to binary files in the directory given as argv[1], where
 * a test compares them with the CPU oracle.  Exit status 0 on success; a
 * library or CUDA error is printed and gives status 1.
 */
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "kvq.h"

enum { B = 2, H = 2, G_RATIO = 4, D = 128, L = 300, MAX_TOKENS = 320, BITS = 4, GROUP = 64 };

static int check_cuda(cudaError_t e, const char *what) {
    if (e != cudaSuccess) {
        fprintf(stderr, "%s: %s\n", what, cudaGetErrorString(e));
        return 1;
    }
    return 0;
}

static int check_kvq(kvq_status s, const char *what) {
    if (s != KVQ_OK) {
        fprintf(stderr, "%s: %s\n", what, kvq_status_string(s));
        return 1;
    }
    return 0;
}

/* fp16 bit patterns of magnitude 2^-4 .. 2^2 with random sign and mantissa
 * (a 64-bit LCG, Knuth's MMIX constants) */
static void fill_f16(uint16_t *x, size_t n, uint64_t *state) {
    for (size_t i = 0; i < n; ++i) {
        *state = *state * 6364136223846793005ull + 1442695040888963407ull;
        const uint32_t r = (uint32_t)(*state >> 33);
        const uint32_t exponent = 11u + (r % 7u);          /* 2^-4 .. 2^2 */
        const uint32_t mantissa = (r >> 3) & 0x3FFu;
        const uint32_t sign = (r >> 13) & 1u;
        x[i] = (uint16_t)((sign << 15) | (exponent << 10) | mantissa);
    }
}

static int write_file(const char *dir, const char *name, const void *p, size_t bytes) {
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE *f = fopen(path, "wb");
    if (f == NULL || fwrite(p, 1, bytes, f) != bytes) {
        fprintf(stderr, "cannot write %s\n", path);
        if (f != NULL) fclose(f);
        return 1;
    }
    fclose(f);
    return 0;
}

int main(int argc, char **argv) {
    if (argc != 2) {
        fprintf(stderr, "usage: %s <output dir>\n", argv[0]);
        return 2;
    }
    const char *dir = argv[1];
    const int q_heads = H * G_RATIO;
    const size_t kv_elems = (size_t)B * H * L * D, q_elems = (size_t)B * q_heads * D;

    uint16_t *k = malloc(kv_elems * 2), *v = malloc(kv_elems * 2), *q = malloc(q_elems * 2);
    float *out = malloc((size_t)B * q_heads * D * 4), *lse = malloc((size_t)B * q_heads * 4);
    if (!k || !v || !q || !out || !lse) return 1;
    uint64_t state = 12345u;
    fill_f16(k, kv_elems, &state);
    fill_f16(v, kv_elems, &state);
    fill_f16(q, q_elems, &state);

    size_t codes_bytes = 0, meta_bytes = 0;
    if (check_kvq(kvq_plane_bytes(B, H, D, MAX_TOKENS, BITS, GROUP, &codes_bytes, &meta_bytes),
                  "kvq_plane_bytes"))
        return 1;

    void *d_k, *d_v, *d_q, *d_kc, *d_km, *d_vc, *d_vm, *d_ws;
    float *d_out, *d_lse;
    int32_t *d_lens;
    if (check_cuda(cudaMalloc(&d_k, kv_elems * 2), "cudaMalloc") ||
        check_cuda(cudaMalloc(&d_v, kv_elems * 2), "cudaMalloc") ||
        check_cuda(cudaMalloc(&d_q, q_elems * 2), "cudaMalloc") ||
        check_cuda(cudaMalloc(&d_kc, codes_bytes), "cudaMalloc") ||
        check_cuda(cudaMalloc(&d_km, meta_bytes), "cudaMalloc") ||
        check_cuda(cudaMalloc(&d_vc, codes_bytes), "cudaMalloc") ||
        check_cuda(cudaMalloc(&d_vm, meta_bytes), "cudaMalloc") ||
        check_cuda(cudaMalloc((void **)&d_out, (size_t)B * q_heads * D * 4), "cudaMalloc") ||
        check_cuda(cudaMalloc((void **)&d_lse, (size_t)B * q_heads * 4), "cudaMalloc") ||
        check_cuda(cudaMalloc((void **)&d_lens, B * 4), "cudaMalloc"))
        return 1;
    if (check_cuda(cudaMemcpy(d_k, k, kv_elems * 2, cudaMemcpyHostToDevice), "copy k") ||
        check_cuda(cudaMemcpy(d_v, v, kv_elems * 2, cudaMemcpyHostToDevice), "copy v") ||
        check_cuda(cudaMemcpy(d_q, q, q_elems * 2, cudaMemcpyHostToDevice), "copy q") ||
        check_cuda(cudaMemset(d_lens, 0, B * 4), "memset lens"))
        return 1;

    kvq_cache cache;
    memset(&cache, 0, sizeof cache);
    cache.batch = B;
    cache.kv_heads = H;
    cache.head_dim = D;
    cache.max_tokens = MAX_TOKENS;
    cache.k.bits = cache.v.bits = BITS;
    cache.k.group_size = cache.v.group_size = GROUP;
    cache.k.fmt = cache.v.fmt = KVQ_FMT_INT;
    cache.k.axis = cache.v.axis = KVQ_AXIS_TOKEN;
    cache.k.codes = d_kc;
    cache.k.meta = d_km;
    cache.v.codes = d_vc;
    cache.v.meta = d_vm;
    cache.seq_lens = d_lens;

    /* the bulk prefill: all L tokens of every (sequence, KV head) */
    if (check_kvq(kvq_quantize_append(&cache, d_k, d_v, KVQ_F16, L, 1, NULL),
                  "kvq_quantize_append"))
        return 1;
    /* ragged lengths for the attention: the full prefill and a shorter one */
    const int32_t lens[B] = {L, 123};
    if (check_cuda(cudaMemcpy(d_lens, lens, sizeof lens, cudaMemcpyHostToDevice), "copy lens"))
        return 1;

    size_t ws_bytes = 0;
    if (check_kvq(kvq_decode_workspace_bytes(&cache, 1, q_heads, MAX_TOKENS, &ws_bytes),
                  "kvq_decode_workspace_bytes") ||
        check_cuda(cudaMalloc(&d_ws, ws_bytes), "cudaMalloc workspace") ||
        check_cuda(cudaMemset(d_ws, 0, ws_bytes), "memset workspace"))
        return 1;
    if (check_kvq(kvq_decode_attention(&cache, 1, d_q, KVQ_F16, q_heads, 1.0f / sqrtf((float)D),
                                       d_out, d_lse, MAX_TOKENS, d_ws, ws_bytes, NULL),
                  "kvq_decode_attention") ||
        check_cuda(cudaDeviceSynchronize(), "synchronize"))
        return 1;

    uint8_t *kc = malloc(codes_bytes), *km = malloc(meta_bytes), *vc = malloc(codes_bytes),
            *vm = malloc(meta_bytes);
    if (!kc || !km || !vc || !vm) return 1;
    if (check_cuda(cudaMemcpy(out, d_out, (size_t)B * q_heads * D * 4, cudaMemcpyDeviceToHost),
                   "copy out") ||
        check_cuda(cudaMemcpy(lse, d_lse, (size_t)B * q_heads * 4, cudaMemcpyDeviceToHost),
                   "copy lse") ||
        check_cuda(cudaMemcpy(kc, d_kc, codes_bytes, cudaMemcpyDeviceToHost), "copy k codes") ||
        check_cuda(cudaMemcpy(km, d_km, meta_bytes, cudaMemcpyDeviceToHost), "copy k meta") ||
        check_cuda(cudaMemcpy(vc, d_vc, codes_bytes, cudaMemcpyDeviceToHost), "copy v codes") ||
        check_cuda(cudaMemcpy(vm, d_vm, meta_bytes, cudaMemcpyDeviceToHost), "copy v meta"))
        return 1;

    if (write_file(dir, "k.bin", k, kv_elems * 2) || write_file(dir, "v.bin", v, kv_elems * 2) ||
        write_file(dir, "q.bin", q, q_elems * 2) ||
        write_file(dir, "out.bin", out, (size_t)B * q_heads * D * 4) ||
        write_file(dir, "lse.bin", lse, (size_t)B * q_heads * 4) ||
        write_file(dir, "k_codes.bin", kc, codes_bytes) ||
        write_file(dir, "k_meta.bin", km, meta_bytes) ||
        write_file(dir, "v_codes.bin", vc, codes_bytes) ||
        write_file(dir, "v_meta.bin", vm, meta_bytes))
        return 1;
    printf("%s: ok (workspace %zu bytes)\n", kvq_version(), ws_bytes);
    return 0;
}
