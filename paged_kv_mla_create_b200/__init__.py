"""Paged MLA decode for B200 (sm_100a): page table, split planner and attention."""
