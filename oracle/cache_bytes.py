"""KV-cache size arithmetic, as the pages state it.  TEST INFRASTRUCTURE ONLY.

The cache holds K and V per layer, each of shape (batch, kv_heads, seq, head_dim),
so its size in bytes is  2 * n_layers * n_kv_heads * d_head * T * b * batch
("Attention variants: MQA, GQA, and MLA", section "The KV cache bill, worked
numerically"; the same product appears in "GQA, MQA, MLA -- Shrinking the
KV-Cache", interview question 4, and per token and layer as h * (d_k + d_v) * 2 in
"Grouped-Query Attention: Fewer KV Heads, Same Quality", section "Counting every
parameter and byte").

The absorbed-MLA cache stores one latent of d_c elements plus a decoupled RoPE key
of d_r elements per token and layer ("Attention variants: MQA, GQA, and MLA",
section "MLA: cache a latent, not the keys and values": d_c + d_r = 576).
"""


def kv_cache_bytes(n_layers, n_kv_heads, head_dim, seq_len, batch=1, bytes_per_elem=2):
    """Bytes of the K and V caches: 2 * L * n_kv * d * T * batch * b."""
    return 2 * n_layers * n_kv_heads * head_dim * seq_len * batch * bytes_per_elem


def kv_bytes_per_token_layer(n_kv_heads, d_k, d_v, bytes_per_elem=2):
    """Per token and layer: n_kv * (d_k + d_v) * b (allows d_k != d_v)."""
    return n_kv_heads * (d_k + d_v) * bytes_per_elem


def mla_cache_bytes(n_layers, d_latent, d_rope, seq_len, batch=1, bytes_per_elem=2):
    """Absorbed-MLA cache: one (d_latent + d_rope)-element row per token and layer."""
    return n_layers * (d_latent + d_rope) * seq_len * batch * bytes_per_elem


def reduction_factor(n_q_heads, n_kv_heads):
    """Cache reduction of GQA against MHA: n_q / n_kv (the pages' boxed h/g)."""
    return n_q_heads / n_kv_heads
