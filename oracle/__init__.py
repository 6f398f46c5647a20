"""CPU oracle for the dMel front end: test infrastructure only (tests, smoke check, CPU baseline)."""
