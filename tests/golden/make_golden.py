"""Writes the golden fixtures in this folder.

Two kinds of values are stored:
  * numbers printed on the pages (the 70-token worked example and the
    block-table figure), typed in with their section named in ``source``;
  * closed forms of softmax(scale * K q) V worked by hand, evaluated here with
    ``math`` only (no page prints an attention example, and nothing here calls
    the CUDA library or the oracle).

Run ``python tests/golden/make_golden.py`` to regenerate.
"""

import json
import math
import os

HERE = os.path.dirname(os.path.abspath(__file__))
E = math.e

FIXTURES = {
    "seventy_tokens.json": {
        "source": "PagedAttention and Continuous Batching (roadtointelligence.com), section "
                  "'Pages, from operating systems', tiny example",
        "statement": "16-token blocks; a request that has produced 70 tokens holds five blocks, "
                     "four full and one with 6 of 16 slots used; at most 15 slots are wasted per "
                     "request",
        "block_size": 16, "tokens": 70, "blocks": 5, "full_blocks": 4, "last_block_used": 6,
        "max_waste_per_request": 15,
    },
    "iteration_level_example.json": {
        "source": "PagedAttention: The vLLM Paper (ai.zenoagi.com), section 'Continuous "
                  "Batching: Request-Level vs. Iteration-Level Scheduling', side-by-side figure; "
                  "also PagedAttention and Continuous Batching (roadtointelligence.com), section "
                  "'Batch by step, not by request'",
        "statement": "with A, B and C in the batch, A finishing lets the waiting D join at the "
                     "next iteration, giving the batch B, C, D; under request-level scheduling D "
                     "would wait until the whole batch is done",
        "reading": "batch of at most 3 sequences; A generates 2 tokens, B and C 4 each, D "
                   "arrives at step 1 and generates 2; one token per request per step",
        "max_num_seqs": 3,
        "requests": [
            {"name": "A", "arrival": 0, "output_len": 2},
            {"name": "B", "arrival": 0, "output_len": 4},
            {"name": "C", "arrival": 0, "output_len": 4},
            {"name": "D", "arrival": 1, "output_len": 2},
        ],
        "iteration_level_batches": [["A", "B", "C"], ["A", "B", "C"], ["B", "C", "D"],
                                    ["B", "C", "D"]],
        "request_level_first_step_of_D": 4,
    },
    "block_table_figure.json": {
        "source": "PagedAttention: The vLLM Paper (ai.zenoagi.com), section 'The Core Idea', GPU "
                  "block pool and block-table figure",
        "statement": "8-block pool B0..B7 holding A-1, B-1, A-2, (empty), B-2, (empty), A-3, B-3; "
                     "request A's table is [0, 2, 6], request B's is [1, 4, 7]; each block holds "
                     "KV for 16 tokens",
        "pool_blocks": 8, "block_size": 16,
        "occupancy": ["A-1", "B-1", "A-2", None, "B-2", None, "A-3", "B-3"],
        "tables": {"A": [0, 2, 6], "B": [1, 4, 7]},
        "free": [3, 5],
    },
    "closed_form_decode.json": {
        "source": "closed forms of softmax(scale * K q) V worked by hand (no page prints an "
                  "attention example)",
        "cases": [
            {"derivation": "x = K q = [1, 0]; p = [e, 1] / (e + 1); "
                           "out = p V = [(e + 3) / (e + 1), (2e + 4) / (e + 1)]",
             "scale": 1.0, "q": [1.0, 0.0], "K": [[1.0, 0.0], [0.0, 0.0]],
             "V": [[1.0, 2.0], [3.0, 4.0]],
             "out": [(E + 3) / (E + 1), (2 * E + 4) / (E + 1)]},
            {"derivation": "x = K q = [0, ln2, 2 ln2]; p = [1, 2, 4] / 7; out = p V = [1, 2]",
             "scale": 1.0, "q": [0.0, math.log(2.0)], "K": [[0.0, 0.0], [0.0, 1.0], [0.0, 2.0]],
             "V": [[7.0, 0.0], [0.0, 7.0], [0.0, 0.0]], "out": [1.0, 2.0]},
            {"derivation": "scale 1/2, x = 0.5 * K q = [0, 0, 0, 0]; uniform p = 1/4; "
                           "out = column means of V = [2.5, -1]",
             "scale": 0.5, "q": [3.0, -1.0, 2.0], "K": [[0.0, 0.0, 0.0]] * 4,
             "V": [[1.0, 0.0], [2.0, -2.0], [3.0, -1.0], [4.0, -1.0]], "out": [2.5, -1.0]},
        ],
    },
}


def main():
    for name, obj in FIXTURES.items():
        with open(os.path.join(HERE, name), "w") as f:
            json.dump(obj, f, indent=1)
            f.write("\n")


if __name__ == "__main__":
    main()
