"""Mutation check of the oracle's pins (CPU only; not collected by pytest).

Each mutant is oracle.c with one plausible mistake planted: a dropped factor, a
wrong index or stride, a swapped operand, a flipped tie rule or bound.  Every
mutant is compiled into a temporary directory (the committed oracle.c and its
library are not touched) and the pins in test_oracle_pins.py are run against it
through the ORACLE_LIB override.  A mutant that no pin rejects is a gap in the
pins; the script lists those and exits 1.

    python tests/oracle_mutants.py [name ...]

Mutants that cannot change any result are left out: for instance, saturating only
values above 464 instead of above 448 in the e4m3 cast changes nothing, since every
value in (448, 464] rounds to 448 anyway.
"""
import os
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path.insert(0, ROOT)

from oracle import build as oracle_build  # noqa: E402

# (name, what the mistake gets wrong, text in oracle.c, replacement)
MUTANTS = [
    ("kv_bytes_no2", "KV bytes per token without the K+V factor 2",
     "return 2 * L * n_kv * d * elt_bytes;", "return L * n_kv * d * elt_bytes;"),
    ("num_blocks_floor1", "block count as floor + 1 instead of the ceiling",
     "return (len + bs - 1) / bs;", "return len / bs + 1;"),
    ("slot_off", "slot offset pos/bs instead of pos%bs",
     "return (int64_t)bt_row[pos / bs] * bs + pos % bs;",
     "return (int64_t)bt_row[pos / bs] * bs + pos / bs;"),
    ("append_headmajor", "append writes a head-major block ([Hkv][bs][d])",
     "int64_t dst = phys * block_stride + (off * Hkv + h) * (int64_t)d;\n                int64_t src",
     "int64_t dst = phys * block_stride + (h * bs + off) * (int64_t)d;\n                int64_t src"),
    ("append_no_stride", "append ignores the block stride",
     "int64_t dst = phys * block_stride + (off * Hkv + h) * (int64_t)d;\n                int64_t src",
     "int64_t dst = phys * ((int64_t)bs * Hkv * d) + (off * Hkv + h) * (int64_t)d;\n"
     "                int64_t src"),
    ("i8_append_no_stride", "INT8 append ignores the block stride",
     "int64_t dst = phys * block_stride + (off * Hkv + h) * (int64_t)d;\n                int64_t sdst",
     "int64_t dst = phys * ((int64_t)bs * Hkv * d) + (off * Hkv + h) * (int64_t)d;\n"
     "                int64_t sdst"),
    ("fp8_append_no_stride", "FP8 append ignores the block stride",
     "int64_t dst = phys * block_stride + (off * Hkv + h) * (int64_t)d;\n"
     "                or_quantize_e4m3(k_new",
     "int64_t dst = phys * ((int64_t)bs * Hkv * d) + (off * Hkv + h) * (int64_t)d;\n"
     "                or_quantize_e4m3(k_new"),
    ("fp8_append_layout", "FP8 append writes a head-major block",
     "int64_t dst = phys * block_stride + (off * Hkv + h) * (int64_t)d;\n"
     "                or_quantize_e4m3(k_new",
     "int64_t dst = phys * block_stride + (h * bs + off) * (int64_t)d;\n"
     "                or_quantize_e4m3(k_new"),
    ("fp8_append_kv_swap", "FP8 append stores V in the K pool and K in the V pool",
     "or_quantize_e4m3(k_new + src, d, k_cache + dst);\n"
     "                or_quantize_e4m3(v_new + src, d, v_cache + dst);",
     "or_quantize_e4m3(v_new + src, d, k_cache + dst);\n"
     "                or_quantize_e4m3(k_new + src, d, v_cache + dst);"),
    ("gather_no_stride", "attention gathers ignore the block stride",
     "int64_t base = phys * block_stride + (off * Hkv + h) * (int64_t)d;\n"
     "            int64_t srow = phys * scale_block_stride + off * Hkv + h; /* scale index */",
     "int64_t base = phys * ((int64_t)bs * Hkv * d) + (off * Hkv + h) * (int64_t)d;\n"
     "            int64_t srow = phys * scale_block_stride + off * Hkv + h; /* scale index */"),
    ("no_scale", "logits without the softmax scale", "s[t] = scale * acc;", "s[t] = acc;"),
    ("softmax_drops_last", "the newest token drops out of the softmax",
     "    for (int t = 0; t < len; ++t) {\n        s[t] = exp(s[t] - m);",
     "    for (int t = 0; t < len; ++t) {\n        s[t] = exp(s[t] - m);\n"
     "        if (t == len - 1 && len > 1) { s[t] = 0.0; }"),
    ("gqa_mod", "query head i reads kv head i % Hkv (interleaved groups)",
     "attend_one(out + ((int64_t)b * Hq + i) * d, qv, Kc, Vc, len, Hkv, i / G, d, scale, s);",
     "attend_one(out + ((int64_t)b * Hq + i) * d, qv, Kc, Vc, len, Hkv, i % Hkv, d, scale, s);"),
    ("v_uses_kscale", "V dequantised with the K scale",
     "Vc[((int64_t)t * Hkv + h) * d + e] = load(v_cache, v_aux,",
     "Vc[((int64_t)t * Hkv + h) * d + e] = load(v_cache, k_aux,"),
    ("i8_decode_sstride", "INT8 decode with a wrong scale-pool block stride",
     "load_int8, block_stride,\n                  (int64_t)bs * Hkv,",
     "load_int8, block_stride,\n                  (int64_t)bs,"),
    ("ratio_squared", "score as the ratio of squared norms",
     "return sqrt(vv) / sqrt(kk);", "return vv / kk;"),
    ("ratio_zero_inf", "||K|| = 0 with ||V|| > 0 scores 0 instead of +inf",
     "if (kk == 0.0) return vv > 0.0 ? INFINITY : 0.0;", "if (kk == 0.0) return 0.0;"),
    ("score_no_stride", "score ignores the block stride",
     "int64_t base = phys * block_stride + (off * Hkv + h) * (int64_t)d;\n"
     "                int64_t srow = phys * scale_block_stride + off * Hkv + h;\n"
     "                double kk",
     "int64_t base = phys * ((int64_t)bs * Hkv * d) + (off * Hkv + h) * (int64_t)d;\n"
     "                int64_t srow = phys * scale_block_stride + off * Hkv + h;\n"
     "                double kk"),
    ("score_i8_scale_stride", "INT8 score with a wrong scale-pool block stride",
     "load_int8, block_stride, (int64_t)bs * Hkv,", "load_int8, block_stride, (int64_t)Hkv,"),
    ("score_i8_swap_scales", "INT8 score with the K and V scale pools swapped",
     "score_common(scores, kq, vq, k_scale, v_scale,", "score_common(scores, kq, vq, v_scale, k_scale,"),
    ("evict_tie_high", "ties in the block argmin go to the highest index",
     "if (best < 0 || mean < best_mean) {", "if (best < 0 || mean <= best_mean) {"),
    ("evict_partial", "the partial newest block is a candidate",
     "int nfull = len / bs;\n        int best = -1;",
     "int nfull = (int)or_num_blocks(len, bs);\n        int best = -1;"),
    ("evict_mean_div", "block mean divided by bs instead of bs*Hkv",
     "double mean = sum / (double)(bs * Hkv);", "double mean = sum / (double)bs;"),
    ("evict_gap_sign", "decision margin with the wrong sign",
     "second == INFINITY) ? INFINITY : second - best_mean;",
     "second == INFINITY) ? INFINITY : best_mean - second;"),
    ("q_128", "INT8 scale amax/128", "volatile float s = amax / 127.0f;",
     "volatile float s = amax / 128.0f;"),
    ("q_roundaway", "INT8 rounding half away from zero",
     "codes[r * d + e] = (int8_t)(int)rintf(y);", "codes[r * d + e] = (int8_t)(int)roundf(y);"),
    ("q_zero_amax", "an all-zero row gets code 1",
     "if (s == 0.0f) {\n                codes[r * d + e] = 0;",
     "if (s == 0.0f) {\n                codes[r * d + e] = 1;"),
    ("i8_append_sdst", "INT8 append stores scales at a wrong index",
     "int64_t sdst = (phys * bs + off) * Hkv + h;", "int64_t sdst = (phys * bs + off) + h;"),
    ("e4m3_sat480", "e4m3 saturates only above 480 (470 becomes the NaN code)",
     "if (a > 448.0) a = 448.0;", "if (a > 480.0) a = 448.0;"),
    ("e4m3_sat_none", "e4m3 without saturation",
     "if (a > 448.0) a = 448.0;", "if (a > 1e300) a = 448.0;"),
    ("e4m3_sub_floor", "e4m3 subnormals truncated",
     "const double m = rint(a * 512.0);", "const double m = floor(a * 512.0);"),
    ("e4m3_round_away", "e4m3 ties away from zero",
     "double m = rint(a / ldexp(1.0, E - 3));", "double m = round(a / ldexp(1.0, E - 3));"),
    ("e4m3_dec_sub", "e4m3 subnormal decode off by a factor 2",
     "ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, E - 7);",
     "ldexp((double)m, -10) : ldexp(1.0 + m / 8.0, E - 7);"),
    ("pf_no_mean", "prefill score summed over heads, not averaged",
     "scores[t] = sum / (double)Hkv;", "scores[t] = sum;"),
    ("pf_tie_earlier", "prefill ties keep the earlier token",
     "return a->i > b->i ? -1 : (a->i < b->i ? 1 : 0);",
     "return a->i < b->i ? -1 : (a->i > b->i ? 1 : 0);"),
    ("pf_nan_top", "NaN scores rank highest",
     "return x != x ? -INFINITY : x;", "return x != x ? INFINITY : x;"),
    ("pf_unsorted", "kept tokens not in prompt order",
     "qsort(row, (size_t)kept, sizeof(int32_t), by_index);", ""),
    ("pack_orig_pos", "kept rows packed at their prompt position",
     "const int64_t slot = or_slot(bt + (int64_t)b * MB, p, bs);",
     "const int64_t slot = or_slot(bt + (int64_t)b * MB, keep_idx[(int64_t)b * budget + p], bs);"),
    ("pack_no_stride", "prefill pack ignores the block stride",
     "const int64_t dst = (slot / bs) * block_stride + (slot % bs) * row;",
     "const int64_t dst = (slot / bs) * (bs * row) + (slot % bs) * row;"),
    ("compact_len1", "compaction shortens the context by 1 instead of bs",
     "ctx_lens[b] -= bs;", "ctx_lens[b] -= 1;"),
    ("compact_partial", "compaction accepts the partial newest block",
     "if (j < 0 || j >= ctx_lens[b] / bs) continue;",
     "if (j < 0 || j >= or_num_blocks(ctx_lens[b], bs)) continue;"),
    ("thr_ge", "threshold policy triggers at exactly 80 %",
     "const int triggered = (double)used_blocks > (1.0 - eviction_ratio) * (double)total_blocks;",
     "const int triggered = (double)used_blocks >= (1.0 - eviction_ratio) * (double)total_blocks;"),
    ("thr_ratio", "trigger at eviction_ratio instead of 1 - eviction_ratio",
     "(1.0 - eviction_ratio) * (double)total_blocks", "eviction_ratio * (double)total_blocks"),
    ("thr_le", "blocks equal to the threshold are evicted",
     "mj == mj && mj < importance_threshold;", "mj == mj && mj <= importance_threshold;"),
    ("thr_no_fallback", "no argmin eviction when no block is below the threshold",
     "if (triggered && n == 0 && argmin[b] >= 0) {", "if (0 && triggered && n == 0 && argmin[b] >= 0) {"),
    ("mask_len", "mask compaction shortens by 1 per block",
     "ctx_lens[b] = len - nf * bs;", "ctx_lens[b] = len - nf;"),
    ("mask_partial", "mask compaction evicts the partial block",
     "if (j < nfull && mask[(int64_t)b * MB + j]) fr[nf++] = row[j];",
     "if (mask[(int64_t)b * MB + j]) fr[nf++] = row[j];"),
    ("pp_excl_self", "chunked prefill: a query does not see its own token",
     "const int upto = bad ? 0 : len - ql + r + 1;", "const int upto = bad ? 0 : len - ql + r;"),
    ("pp_noncausal", "chunked prefill without the causal mask",
     "const int upto = bad ? 0 : len - ql + r + 1;", "const int upto = bad ? 0 : len;"),
    ("pp_bad_ql", "q_len > context not treated as invalid",
     "const int bad = len < 0 || (int64_t)len > (int64_t)MB * bs || ql > len;",
     "const int bad = len < 0 || (int64_t)len > (int64_t)MB * bs;"),
    ("pp_gqa", "chunked prefill with interleaved GQA groups",
     "attend_one(out + (row * Hq + i) * d, qv, Kc, Vc, upto, Hkv, i / G, d, scale, s);",
     "attend_one(out + (row * Hq + i) * d, qv, Kc, Vc, upto, Hkv, i % Hkv, d, scale, s);"),
    ("pp_q_index", "chunked prefill reads q rows without the sequence offset",
     "qv[e] = bf16_to_f64(q[(row * Hq + i) * d + e]);",
     "qv[e] = bf16_to_f64(q[((int64_t)r * Hq + i) * d + e]);"),
]


def main(only) -> int:
    src = open(oracle_build.SRC).read()
    survivors, broken = [], []
    with tempfile.TemporaryDirectory() as tmp:
        for name, what, find, repl in MUTANTS:
            if only and name not in only:
                continue
            if src.count(find) != 1:
                broken.append(name)
                print(f"{name:24s} text not found once in oracle.c", flush=True)
                continue
            msrc = os.path.join(tmp, name + ".c")
            mlib = os.path.join(tmp, name + ".so")
            with open(msrc, "w") as f:
                f.write(src.replace(find, repl))
            oracle_build.compile_c(msrc, mlib, extra=("-w",))
            env = dict(os.environ, ORACLE_LIB=mlib)
            r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                                os.path.join(HERE, "test_oracle_pins.py")],
                               cwd=ROOT, env=env, capture_output=True, text=True)
            caught = r.returncode != 0
            if not caught:
                survivors.append(name)
            print(f"{name:24s} {'caught' if caught else 'SURVIVED'}  {what}", flush=True)
    print(f"{len(MUTANTS) if not only else len(only)} mutants; survivors: {survivors}; "
          f"stale: {broken}")
    return 1 if survivors or broken else 0


if __name__ == "__main__":
    sys.exit(main(set(sys.argv[1:])))
