"""fp64 CPU oracle for ragged paged attention -- test infrastructure only.

Imported by the tests, by ``__graft_entry__.smoke()`` and by the benchmark's CPU-baseline
leg; never by the library.  See ``rpa_oracle`` for what each function computes and the
passage it follows.
"""
from .rpa_oracle import (SEQ_MAJOR, HEAD_MAJOR, attend_row, attention, bits16,
                         build_group_tables, forward, logical_rows, merge_partials,
                         seq_ranges, visible_keys, widen, write_kv)

__all__ = ["SEQ_MAJOR", "HEAD_MAJOR", "attend_row", "attention", "bits16",
           "build_group_tables", "forward", "logical_rows", "merge_partials", "seq_ranges",
           "visible_keys", "widen", "write_kv"]
