/*
 * A plain C consumer of the kvq C ABI (include/kvq.h): compiled as C11 and
 * linked against libkvq.so, it calls the entry points that need no GPU --
 * sizes, k, descriptor validation -- and prints one result per line for the
 * test that builds it to compare.
 */
#include <stdio.h>
#include <string.h>

#include "kvq.h"

int main(void)
{
    printf("version %d\n", kvq_version());
    printf("page_bytes %zu %zu %zu %zu\n", kvq_page_bytes(2, 32), kvq_page_bytes(4, 32),
           kvq_page_bytes(2, 128), kvq_page_bytes(3, 32));
    printf("num_selected %d %d %d %d\n", kvq_num_selected(0.0f, 128), kvq_num_selected(0.4f, 128),
           kvq_num_selected(0.6f, 128), kvq_num_selected(1.0f, 128));
    printf("status_words %zu\n", kvq_status_words(2, 8));

    kvq_cache c;
    memset(&c, 0, sizeof c);
    c.batch = 2;
    c.n_kv_heads = 8;
    c.head_dim = 128;
    c.group = 32;
    c.bits = 2;
    c.capacity = 256;
    printf("cache_bytes %zu\n", kvq_cache_bytes(&c));
    c.n_sink = 64;
    c.n_recent = 256;
    c.group = 128;
    printf("cache_bytes_tier %zu\n", kvq_cache_bytes(&c));
    c.bucket = 128;
    printf("num_buckets %d\n", kvq_num_buckets(&c));

    /* argument errors are caught on the host, before anything is launched */
    printf("append_null %d\n", kvq_append(NULL, NULL, NULL, KVQ_DTYPE_BF16, 1, NULL, NULL));
    printf("init_null %d\n", kvq_cache_init(&c, NULL));
    printf("copy_null %d\n", kvq_copy_async(NULL, NULL, 16, NULL));
    printf("string %s\n", kvq_status_string(KVQ_ERR_CAPACITY));
    return 0;
}
