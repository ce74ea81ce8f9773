/*
 * A plain C99 consumer of llama_fwd.h: it must compile with -std=c99 -pedantic
 * and link against liblfwd.so. It exercises only host-side paths (argument and
 * config checks, error messages), so it runs without a GPU; it prints "ok" and
 * returns 0 when every check holds, else names the first failing one.
 */
#include <stdio.h>
#include <string.h>

#include "llama_fwd.h"

#define CHECK(cond)                                         \
    do {                                                    \
        if (!(cond)) {                                      \
            printf("failed: %s (line %d)\n", #cond, __LINE__); \
            return 1;                                       \
        }                                                   \
    } while (0)

int main(void) {
    llm_model* m = NULL;
    llm_config cfg;
    llm_weights w;
    int64_t strides[4];
    void *k = NULL, *v = NULL;
    memset(&cfg, 0, sizeof cfg);
    memset(&w, 0, sizeof w);

    CHECK(llm_model_init(NULL, NULL, NULL, &m) == LLM_ERR_NULL_PTR);
    CHECK(m == NULL);
    CHECK(strstr(llm_last_error(), "NULL") != NULL);

    /* the Llama-3-8B config with one KV head (multi-query) and no weights:
       the config is valid, the missing weights are reported */
    cfg.dim = 4096; cfg.n_layers = 32; cfg.n_heads = 32; cfg.n_kv_heads = 1; cfg.head_dim = 128;
    cfg.ffn_hidden = 14336; cfg.vocab = 128256; cfg.max_seq_len = 8192; cfg.max_batch = 1;
    cfg.norm_eps = 1e-5f; cfg.rope_theta = 500000.0f; cfg.dtype = LLM_BF16;
    cfg.has_embed_and_head = 1;
    CHECK(llm_model_init(&cfg, &w, NULL, &m) == LLM_ERR_NULL_PTR);
    CHECK(strstr(llm_last_error(), "weight") != NULL);
    cfg.n_kv_heads = 5;  /* does not divide n_heads */
    CHECK(llm_model_init(&cfg, &w, NULL, &m) == LLM_ERR_BAD_CONFIG);
    cfg.n_kv_heads = 8;
    cfg.max_batch = 17;
    CHECK(llm_model_init(&cfg, &w, NULL, &m) == LLM_ERR_BAD_CONFIG);

    CHECK(llm_prefill(NULL, NULL, 1, 1, NULL, NULL) == LLM_ERR_NULL_PTR);
    CHECK(llm_decode_step(NULL, 1, NULL, NULL, NULL) == LLM_ERR_NULL_PTR);
    CHECK(llm_kv_cache_reset(NULL) == LLM_ERR_NULL_PTR);
    CHECK(llm_kv_cache_view(NULL, &k, &v, strides) == LLM_ERR_NULL_PTR);
    CHECK(llm_synchronize(NULL) == LLM_ERR_NULL_PTR);
    llm_model_free(NULL);

    CHECK(llm_op_attention_decode_workspace(1, 1, 32, 8, 128) > 0);
    CHECK(llm_op_attention_decode_workspace(1, 1, 30, 8, 128) == 0);
    CHECK(llm_op_gemv_workspace(4096, 4096) > 0);
    printf("ok\n");
    return 0;
}
